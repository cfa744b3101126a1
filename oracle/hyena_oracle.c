/*
 * hyena_oracle.c -- plain float64 CPU oracle for the Hyena long-convolution
 * operator (filter generation, causal long convolution, order-N gated
 * recurrence, and the 2-D variant).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product (CUDA)
 * path never links, loads or calls it, and the two share no code, header,
 * table or constant generator.
 *
 * Sources (page title, section):
 *  - "Hyena Hierarchy: Towards Larger Convolutional Language Models",
 *    abstract: the operator interleaves implicitly parametrised long
 *    convolutions with data-controlled (multiplicative) gating.  This file
 *    reads that as the order-N recurrence
 *        z_0 = v,   z_n = x_n * (h_n (*) z_{n-1} + b_n * z_{n-1}),   y = z_N
 *    with (*) a per-channel causal convolution over the whole sequence and
 *    b_n a per-channel bias (skip) term.
 *  - "Long Context Language Models and their Biological Applications with
 *    Eric Nguyen - #690", 4:29 (an MLP parametrises the filter), 5:48 (the
 *    filter is as long as the input: a global convolution), 6:27 (the
 *    convolution theorem: FFT both, multiply elementwise, transform back).
 *  - "Native Multi-Dimensional Subquadratic Operators via Input Dependent
 *    Long Convolutions", Methodology, "Native ND Convolution" (N-D FFT on the
 *    grid) and "Handling Boundaries" (non-circular convolution by zero
 *    padding to double the grid before the FFT).
 *
 * Readings where the pages are silent (the pages give no formulas):
 *  - conv(h, u)[t] = sum_{s=0..t} h[s] u[t-s]: h[0] is the zero-lag tap,
 *    no flip, no centring; the result is causal.
 *  - The filter network: features phi(i) = [t, sin(2 pi k t), cos(2 pi k t)
 *    for k = 1..K], t = i/L; three bias-free Linear+sin layers of the given
 *    width; one bias-free linear head to N*D outputs; filter n, channel d is
 *    head row n*D + d; times the window exp(-alpha_d * t * L / decay_div).
 *  - 2-D: features [ty, tx, sin/cos(2 pi k ty) for k = 1..K,
 *    sin/cos(2 pi k tx) for k = 1..K], ty = iy/H, tx = ix/W; the same FFN;
 *    separable window exp(-alpha_c ty H / div) * exp(-alpha_c tx W / div).
 *
 * Every routine is written for clarity, not speed: loops in the order of the
 * definition, a textbook iterative radix-2 FFT whose twiddles are taken
 * from cos/sin of each angle in float64, no blocking, no fusion.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_PI 3.14159265358979323846

enum { ORACLE_OK = 0, ORACLE_EBADARG = -1, ORACLE_ENOMEM = -2 };
enum { ROUTE_DIRECT = 0, ROUTE_FFT = 1 };

static int is_pow2(long n) { return n > 0 && (n & (n - 1)) == 0; }

static long next_pow2(long n)
{
    long p = 1;
    while (p < n) p <<= 1;
    return p;
}

/* ------------------------------------------------------------------ */
/* Filter network (TWIML #690, 4:29: an MLP parametrises the filter).  */
/* ------------------------------------------------------------------ */

/* out[r] = sum_c W[r][c] * in[c]   (W row-major [rows][cols]) */
static void matvec(const double *W, int rows, int cols, const double *in,
                   double *out)
{
    for (int r = 0; r < rows; ++r) {
        double s = 0.0;
        for (int c = 0; c < cols; ++c) s += W[(long)r * cols + c] * in[c];
        out[r] = s;
    }
}

/* The FFN: three Linear+sin layers then a linear head. */
static void ffn(const double *W1, const double *W2, const double *W3,
                const double *Wout, int n_in, int width, int n_out,
                const double *phi, double *a1, double *a2, double *a3,
                double *o)
{
    matvec(W1, width, n_in, phi, a1);
    for (int j = 0; j < width; ++j) a1[j] = sin(a1[j]);
    matvec(W2, width, width, a1, a2);
    for (int j = 0; j < width; ++j) a2[j] = sin(a2[j]);
    matvec(W3, width, width, a2, a3);
    for (int j = 0; j < width; ++j) a3[j] = sin(a3[j]);
    matvec(Wout, n_out, width, a3, o);
}

typedef struct {
    const double *W1, *W2, *W3, *Wout, *alpha;
    int N, D, L, n_bands, width;
    double decay_div;
    double *h;
    int i0, i1; /* positions handled by this worker */
    int status;
} fg_job;

static void *filter_gen_worker(void *arg)
{
    fg_job *j = (fg_job *)arg;
    const int n_in = 1 + 2 * j->n_bands;
    const int n_out = j->N * j->D;
    double *phi = malloc(sizeof(double) * n_in);
    double *a1 = malloc(sizeof(double) * j->width);
    double *a2 = malloc(sizeof(double) * j->width);
    double *a3 = malloc(sizeof(double) * j->width);
    double *o = malloc(sizeof(double) * n_out);
    if (!phi || !a1 || !a2 || !a3 || !o) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (int i = j->i0; i < j->i1; ++i) {
        const double t = (double)i / (double)j->L;
        phi[0] = t;
        for (int k = 1; k <= j->n_bands; ++k) {
            phi[2 * k - 1] = sin(2.0 * ORACLE_PI * k * t);
            phi[2 * k] = cos(2.0 * ORACLE_PI * k * t);
        }
        ffn(j->W1, j->W2, j->W3, j->Wout, n_in, j->width, n_out, phi, a1, a2,
            a3, o);
        for (int n = 0; n < j->N; ++n)
            for (int d = 0; d < j->D; ++d) {
                const double window =
                    exp(-j->alpha[d] * t * (double)j->L / j->decay_div);
                j->h[((long)n * j->D + d) * j->L + i] = o[n * j->D + d] * window;
            }
    }
    j->status = ORACLE_OK;
done:
    free(phi); free(a1); free(a2); free(a3); free(o);
    return NULL;
}

/* h[N][D][L] from the FFN weights (W1 [width][1+2K], W2, W3 [width][width],
 * Wout [N*D][width], all row-major [out][in]) and the decay rates alpha[D]. */
int oracle_filter_gen(const double *W1, const double *W2, const double *W3,
                      const double *Wout, const double *alpha, int N, int D,
                      int L, int n_bands, int width, double decay_div,
                      int nthreads, double *h)
{
    if (!W1 || !W2 || !W3 || !Wout || !alpha || !h || N < 1 || D < 1 ||
        L < 1 || n_bands < 0 || width < 1 || !(decay_div > 0.0))
        return ORACLE_EBADARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > L) nthreads = L;
    fg_job *jobs = calloc(nthreads, sizeof(fg_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fg_job j = {W1, W2, W3, Wout, alpha, N, D, L, n_bands, width,
                    decay_div, h, (int)((long)L * k / nthreads),
                    (int)((long)L * (k + 1) / nthreads), 0};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, filter_gen_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* ------------------------------------------------------------------ */
/* Input-dependent filters ("Native Multi-Dimensional Subquadratic       */
/* Operators via Input Dependent Long Convolutions": Input-Dependent     */
/* Kernels via Registers and FiLM; Kernel Parameterization).             */
/* ------------------------------------------------------------------ */
/*
 * Per sample b the sine layers are modulated feature-wise (FiLM) by the
 * sample's control vectors, and each hidden unit has its own frequency:
 *     a_l = sin(omega_l * (gamma_{b,l} * (W_l a_{l-1}) + beta_{b,l})),
 * l = 1..3, then o = Wout a_3; the filter is o times a window: the
 * exponential decay exp(-alpha_d t L / div) of the shared filters, or the
 * Gaussian exp(-t^2 / (2 sigma_d^2)), t = i/L.  The control vectors come
 * from the sample (the pages derive them from register tokens); here they
 * are inputs.  omega = 1, gamma = 1, beta = 0 with the exponential window
 * is the shared filter of oracle_filter_gen.
 */
typedef struct {
    const double *W1, *W2, *W3, *Wout, *omega, *gamma, *beta, *win;
    int gaussian, B, N, D, L, n_bands, width;
    double decay_div;
    double *h;
    int i0, i1;
    int status;
} fgf_job;

/* a[j] = sin(om[j] * (g[j] * a[j] + be[j])) */
static void film_sin(double *a, int width, const double *om, const double *g, const double *be)
{
    for (int j = 0; j < width; ++j) a[j] = sin(om[j] * (g[j] * a[j] + be[j]));
}

static void *filter_gen_film_worker(void *arg)
{
    fgf_job *j = (fgf_job *)arg;
    const int n_in = 1 + 2 * j->n_bands, w = j->width, n_out = j->N * j->D;
    double *phi = malloc(sizeof(double) * n_in);
    double *a1 = malloc(sizeof(double) * w), *a2 = malloc(sizeof(double) * w);
    double *a3 = malloc(sizeof(double) * w), *o = malloc(sizeof(double) * n_out);
    if (!phi || !a1 || !a2 || !a3 || !o) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (int b = 0; b < j->B; ++b) {
        const double *g = j->gamma + (long)b * 3 * w, *be = j->beta + (long)b * 3 * w;
        for (int i = j->i0; i < j->i1; ++i) {
            const double t = (double)i / (double)j->L;
            phi[0] = t;
            for (int k = 1; k <= j->n_bands; ++k) {
                phi[2 * k - 1] = sin(2.0 * ORACLE_PI * k * t);
                phi[2 * k] = cos(2.0 * ORACLE_PI * k * t);
            }
            matvec(j->W1, w, n_in, phi, a1);
            film_sin(a1, w, j->omega, g, be);
            matvec(j->W2, w, w, a1, a2);
            film_sin(a2, w, j->omega + w, g + w, be + w);
            matvec(j->W3, w, w, a2, a3);
            film_sin(a3, w, j->omega + 2 * w, g + 2 * w, be + 2 * w);
            matvec(j->Wout, n_out, w, a3, o);
            for (int n = 0; n < j->N; ++n)
                for (int d = 0; d < j->D; ++d) {
                    const double window =
                        j->gaussian ? exp(-t * t / (2.0 * j->win[d] * j->win[d]))
                                    : exp(-j->win[d] * t * (double)j->L / j->decay_div);
                    j->h[(((long)b * j->N + n) * j->D + d) * j->L + i] = o[n * j->D + d] * window;
                }
        }
    }
    j->status = ORACLE_OK;
done:
    free(phi); free(a1); free(a2); free(a3); free(o);
    return NULL;
}

/* h[B][N][D][L]: per-sample filters.  omega [3][width], gamma and beta
 * [B][3][width]; win [D] is alpha (gaussian = 0) or sigma (gaussian = 1). */
int oracle_filter_gen_film(const double *W1, const double *W2, const double *W3,
                           const double *Wout, const double *omega, const double *gamma,
                           const double *beta, const double *win, int gaussian, int B, int N,
                           int D, int L, int n_bands, int width, double decay_div,
                           int nthreads, double *h)
{
    if (!W1 || !W2 || !W3 || !Wout || !omega || !gamma || !beta || !win || !h || B < 1 ||
        N < 1 || D < 1 || L < 1 || n_bands < 0 || width < 1 || !(decay_div > 0.0))
        return ORACLE_EBADARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > L) nthreads = L;
    fgf_job *jobs = calloc(nthreads, sizeof(fgf_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fgf_job j = {W1, W2, W3, Wout, omega, gamma, beta, win, gaussian, B, N, D, L, n_bands,
                     width, decay_div, h, (int)((long)L * k / nthreads),
                     (int)((long)L * (k + 1) / nthreads), 0};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, filter_gen_film_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

typedef struct {
    const double *W1, *W2, *W3, *Wout, *alpha;
    int N, C, H, W, n_bands, width;
    double decay_div;
    double *h;
    int p0, p1; /* flattened grid positions handled by this worker */
    int status;
} fg2_job;

static void *filter_gen_2d_worker(void *arg)
{
    fg2_job *j = (fg2_job *)arg;
    const int n_in = 2 + 4 * j->n_bands;
    const int n_out = j->N * j->C;
    const long HW = (long)j->H * j->W;
    double *phi = malloc(sizeof(double) * n_in);
    double *a1 = malloc(sizeof(double) * j->width);
    double *a2 = malloc(sizeof(double) * j->width);
    double *a3 = malloc(sizeof(double) * j->width);
    double *o = malloc(sizeof(double) * n_out);
    if (!phi || !a1 || !a2 || !a3 || !o) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (int p = j->p0; p < j->p1; ++p) {
        const int iy = p / j->W, ix = p % j->W;
        const double ty = (double)iy / (double)j->H;
        const double tx = (double)ix / (double)j->W;
        phi[0] = ty;
        phi[1] = tx;
        for (int k = 1; k <= j->n_bands; ++k) {
            phi[2 * k] = sin(2.0 * ORACLE_PI * k * ty);
            phi[2 * k + 1] = cos(2.0 * ORACLE_PI * k * ty);
        }
        for (int k = 1; k <= j->n_bands; ++k) {
            phi[2 * j->n_bands + 2 * k] = sin(2.0 * ORACLE_PI * k * tx);
            phi[2 * j->n_bands + 2 * k + 1] = cos(2.0 * ORACLE_PI * k * tx);
        }
        ffn(j->W1, j->W2, j->W3, j->Wout, n_in, j->width, n_out, phi, a1, a2,
            a3, o);
        for (int n = 0; n < j->N; ++n)
            for (int c = 0; c < j->C; ++c) {
                const double window =
                    exp(-j->alpha[c] * ty * (double)j->H / j->decay_div) *
                    exp(-j->alpha[c] * tx * (double)j->W / j->decay_div);
                j->h[((long)n * j->C + c) * HW + p] = o[n * j->C + c] * window;
            }
    }
    j->status = ORACLE_OK;
done:
    free(phi); free(a1); free(a2); free(a3); free(o);
    return NULL;
}

/* Input-dependent 2-D filters: the FiLM-modulated sine layers of
 * oracle_filter_gen_film on the 2-D features, h[B][N][C][H][W]; the
 * window is the separable exponential decay of oracle_filter_gen_2d
 * (gaussian = 0, win = alpha) or the Gaussian exp(-(ty^2 + tx^2) /
 * (2 sigma_c^2)) (gaussian = 1, win = sigma). */
typedef struct {
    const double *W1, *W2, *W3, *Wout, *omega, *gamma, *beta, *win;
    int gaussian, B, N, C, H, W, n_bands, width;
    double decay_div;
    double *h;
    int p0, p1;
    int status;
} fgf2_job;

static void *filter_gen_film_2d_worker(void *arg)
{
    fgf2_job *j = (fgf2_job *)arg;
    const int n_in = 2 + 4 * j->n_bands, w = j->width, n_out = j->N * j->C;
    const long HW = (long)j->H * j->W;
    double *phi = malloc(sizeof(double) * n_in);
    double *a1 = malloc(sizeof(double) * w), *a2 = malloc(sizeof(double) * w);
    double *a3 = malloc(sizeof(double) * w), *o = malloc(sizeof(double) * n_out);
    if (!phi || !a1 || !a2 || !a3 || !o) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (int b = 0; b < j->B; ++b) {
        const double *g = j->gamma + (long)b * 3 * w, *be = j->beta + (long)b * 3 * w;
        for (int p = j->p0; p < j->p1; ++p) {
            const int iy = p / j->W, ix = p % j->W;
            const double ty = (double)iy / (double)j->H, tx = (double)ix / (double)j->W;
            phi[0] = ty;
            phi[1] = tx;
            for (int k = 1; k <= j->n_bands; ++k) {
                phi[2 * k] = sin(2.0 * ORACLE_PI * k * ty);
                phi[2 * k + 1] = cos(2.0 * ORACLE_PI * k * ty);
                phi[2 * j->n_bands + 2 * k] = sin(2.0 * ORACLE_PI * k * tx);
                phi[2 * j->n_bands + 2 * k + 1] = cos(2.0 * ORACLE_PI * k * tx);
            }
            matvec(j->W1, w, n_in, phi, a1);
            film_sin(a1, w, j->omega, g, be);
            matvec(j->W2, w, w, a1, a2);
            film_sin(a2, w, j->omega + w, g + w, be + w);
            matvec(j->W3, w, w, a2, a3);
            film_sin(a3, w, j->omega + 2 * w, g + 2 * w, be + 2 * w);
            matvec(j->Wout, n_out, w, a3, o);
            for (int n = 0; n < j->N; ++n)
                for (int c = 0; c < j->C; ++c) {
                    const double s = j->win[c];
                    const double window =
                        j->gaussian ? exp(-(ty * ty + tx * tx) / (2.0 * s * s))
                                    : exp(-s * ty * (double)j->H / j->decay_div) *
                                          exp(-s * tx * (double)j->W / j->decay_div);
                    j->h[(((long)b * j->N + n) * j->C + c) * HW + p] = o[n * j->C + c] * window;
                }
        }
    }
    j->status = ORACLE_OK;
done:
    free(phi); free(a1); free(a2); free(a3); free(o);
    return NULL;
}

int oracle_filter_gen_film_2d(const double *W1, const double *W2, const double *W3,
                              const double *Wout, const double *omega, const double *gamma,
                              const double *beta, const double *win, int gaussian, int B, int N,
                              int C, int H, int W, int n_bands, int width, double decay_div,
                              int nthreads, double *h)
{
    if (!W1 || !W2 || !W3 || !Wout || !omega || !gamma || !beta || !win || !h || B < 1 ||
        N < 1 || C < 1 || H < 1 || W < 1 || n_bands < 0 || width < 1 || !(decay_div > 0.0))
        return ORACLE_EBADARG;
    const int HW = H * W;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > HW) nthreads = HW;
    fgf2_job *jobs = calloc(nthreads, sizeof(fgf2_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fgf2_job j = {W1, W2, W3, Wout, omega, gamma, beta, win, gaussian, B, N, C, H, W, n_bands,
                      width, decay_div, h, (int)((long)HW * k / nthreads),
                      (int)((long)HW * (k + 1) / nthreads), 0};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, filter_gen_film_2d_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* h[N][C][H][W] from the FFN weights (W1 [width][2+4K]) and alpha[C]. */
int oracle_filter_gen_2d(const double *W1, const double *W2, const double *W3,
                         const double *Wout, const double *alpha, int N, int C,
                         int H, int W, int n_bands, int width,
                         double decay_div, int nthreads, double *h)
{
    if (!W1 || !W2 || !W3 || !Wout || !alpha || !h || N < 1 || C < 1 ||
        H < 1 || W < 1 || n_bands < 0 || width < 1 || !(decay_div > 0.0))
        return ORACLE_EBADARG;
    const int HW = H * W;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > HW) nthreads = HW;
    fg2_job *jobs = calloc(nthreads, sizeof(fg2_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fg2_job j = {W1, W2, W3, Wout, alpha, N, C, H, W, n_bands, width,
                     decay_div, h, (int)((long)HW * k / nthreads),
                     (int)((long)HW * (k + 1) / nthreads), 0};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, filter_gen_2d_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* ------------------------------------------------------------------ */
/* Naive iterative radix-2 FFT (TWIML #690, 6:27: the FFT route).      */
/* ------------------------------------------------------------------ */

/* In place, unnormalised: X[k] = sum_j x[j] exp(sign * 2 pi i j k / n).
 * sign = -1 is the forward transform.  n must be a power of two. */
static void fft_radix2(double *re, double *im, long n, int sign)
{
    /* bit-reversal permutation */
    for (long i = 1, j = 0; i < n; ++i) {
        long bit = n >> 1;
        for (; j & bit; bit >>= 1) j ^= bit;
        j ^= bit;
        if (i < j) {
            double t = re[i]; re[i] = re[j]; re[j] = t;
            t = im[i]; im[i] = im[j]; im[j] = t;
        }
    }
    /* log2(n) butterfly stages; the twiddle of each butterfly comes from
     * cos/sin of its own angle */
    for (long len = 2; len <= n; len <<= 1) {
        const long half = len / 2;
        for (long k = 0; k < half; ++k) {
            const double ang = sign * 2.0 * ORACLE_PI * (double)k / (double)len;
            const double wr = cos(ang), wi = sin(ang);
            for (long s = 0; s < n; s += len) {
                const long a = s + k, b = a + half;
                const double tr = wr * re[b] - wi * im[b];
                const double ti = wr * im[b] + wi * re[b];
                re[b] = re[a] - tr;
                im[b] = im[a] - ti;
                re[a] += tr;
                im[a] += ti;
            }
        }
    }
}

/* Exposed for the oracle's own pins (closed forms, Parseval). */
int oracle_fft(double *re, double *im, long n, int sign)
{
    if (!re || !im || !is_pow2(n) || (sign != 1 && sign != -1))
        return ORACLE_EBADARG;
    fft_radix2(re, im, n, sign);
    return ORACLE_OK;
}

/* Spectrum of each row of h[rows][L] zero-padded to P = 2L (Handling
 * Boundaries: pad to double the grid).  Keeps bins 0..L of the P-point DFT:
 * out_re/out_im [rows][L+1].  P must be a power of two. */
int oracle_rfft_pad2(const double *h, long rows, long L, double *out_re,
                     double *out_im)
{
    const long P = 2 * L;
    if (!h || !out_re || !out_im || rows < 0 || L < 1 || !is_pow2(P))
        return ORACLE_EBADARG;
    double *re = malloc(sizeof(double) * P), *im = malloc(sizeof(double) * P);
    if (!re || !im) { free(re); free(im); return ORACLE_ENOMEM; }
    for (long r = 0; r < rows; ++r) {
        for (long t = 0; t < P; ++t) {
            re[t] = t < L ? h[r * L + t] : 0.0;
            im[t] = 0.0;
        }
        fft_radix2(re, im, P, -1);
        for (long k = 0; k <= L; ++k) {
            out_re[r * (L + 1) + k] = re[k];
            out_im[r * (L + 1) + k] = im[k];
        }
    }
    free(re); free(im);
    return ORACLE_OK;
}

/* 2-D spectrum of each h[rows][H][W] zero-padded to 2H x 2W; keeps
 * columns 0..W of every one of the 2H rows: out [rows][2H][W+1]. */
int oracle_rfft2_pad2(const double *h, long rows, long H, long W,
                      double *out_re, double *out_im)
{
    const long PH = 2 * H, PW = 2 * W;
    if (!h || !out_re || !out_im || rows < 0 || H < 1 || W < 1 ||
        !is_pow2(PH) || !is_pow2(PW))
        return ORACLE_EBADARG;
    double *re = malloc(sizeof(double) * PH * PW);
    double *im = malloc(sizeof(double) * PH * PW);
    double *cr = malloc(sizeof(double) * PH), *ci = malloc(sizeof(double) * PH);
    if (!re || !im || !cr || !ci) {
        free(re); free(im); free(cr); free(ci);
        return ORACLE_ENOMEM;
    }
    for (long r = 0; r < rows; ++r) {
        for (long y = 0; y < PH; ++y)
            for (long x = 0; x < PW; ++x) {
                re[y * PW + x] = (y < H && x < W) ? h[(r * H + y) * W + x] : 0.0;
                im[y * PW + x] = 0.0;
            }
        for (long y = 0; y < PH; ++y) fft_radix2(re + y * PW, im + y * PW, PW, -1);
        for (long x = 0; x < PW; ++x) {
            for (long y = 0; y < PH; ++y) { cr[y] = re[y * PW + x]; ci[y] = im[y * PW + x]; }
            fft_radix2(cr, ci, PH, -1);
            for (long y = 0; y < PH; ++y) { re[y * PW + x] = cr[y]; im[y * PW + x] = ci[y]; }
        }
        for (long y = 0; y < PH; ++y)
            for (long x = 0; x <= W; ++x) {
                out_re[(r * PH + y) * (W + 1) + x] = re[y * PW + x];
                out_im[(r * PH + y) * (W + 1) + x] = im[y * PW + x];
            }
    }
    free(re); free(im); free(cr); free(ci);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Causal long convolution, two independent routes.                   */
/* ------------------------------------------------------------------ */

/* The definition: y[t] = sum_{s=0..t} h[s] u[t-s]. */
static void conv_direct(const double *h, const double *u, long L, double *y)
{
    for (long t = 0; t < L; ++t) {
        double s = 0.0;
        for (long k = 0; k <= t; ++k) s += h[k] * u[t - k];
        y[t] = s;
    }
}

typedef struct { double *hr, *hi, *ur, *ui; long P; } fft_scratch;

static int scratch_alloc(fft_scratch *s, long P)
{
    s->P = P;
    s->hr = malloc(sizeof(double) * P); s->hi = malloc(sizeof(double) * P);
    s->ur = malloc(sizeof(double) * P); s->ui = malloc(sizeof(double) * P);
    return (s->hr && s->hi && s->ur && s->ui) ? ORACLE_OK : ORACLE_ENOMEM;
}

static void scratch_free(fft_scratch *s)
{
    free(s->hr); free(s->hi); free(s->ur); free(s->ui);
}

/* The convolution theorem route: zero-pad h and u to P >= 2L (a power of
 * two, so no wrap-around reaches t < L), DFT both, multiply, inverse DFT,
 * scale by 1/P, keep t < L. */
static void conv_fft(const double *h, const double *u, long L, double *y,
                     fft_scratch *s)
{
    const long P = s->P;
    for (long t = 0; t < P; ++t) {
        s->hr[t] = t < L ? h[t] : 0.0; s->hi[t] = 0.0;
        s->ur[t] = t < L ? u[t] : 0.0; s->ui[t] = 0.0;
    }
    fft_radix2(s->hr, s->hi, P, -1);
    fft_radix2(s->ur, s->ui, P, -1);
    for (long k = 0; k < P; ++k) {
        const double re = s->hr[k] * s->ur[k] - s->hi[k] * s->ui[k];
        const double im = s->hr[k] * s->ui[k] + s->hi[k] * s->ur[k];
        s->ur[k] = re;
        s->ui[k] = im;
    }
    fft_radix2(s->ur, s->ui, P, +1);
    for (long t = 0; t < L; ++t) y[t] = s->ur[t] / (double)P;
}

int oracle_conv(const double *h, const double *u, long L, int route, double *y)
{
    if (!h || !u || !y || L < 1) return ORACLE_EBADARG;
    if (route == ROUTE_DIRECT) {
        conv_direct(h, u, L, y);
        return ORACLE_OK;
    }
    if (route != ROUTE_FFT) return ORACLE_EBADARG;
    fft_scratch s;
    if (scratch_alloc(&s, next_pow2(2 * L)) != ORACLE_OK) {
        scratch_free(&s);
        return ORACLE_ENOMEM;
    }
    conv_fft(h, u, L, y, &s);
    scratch_free(&s);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* Circular convolution ("Native Multi-Dimensional Subquadratic         */
/* Operators ...", Handling Boundaries: circular convolutions for        */
/* periodic systems, the alternative to zero padding).                   */
/* ------------------------------------------------------------------ */

/* The definition: y[t] = sum_{s=0..L-1} h[s] u[(t - s) mod L]. */
static void cconv_direct(const double *h, const double *u, long L, double *y)
{
    for (long t = 0; t < L; ++t) {
        double s = 0.0;
        for (long k = 0; k < L; ++k) s += h[k] * u[((t - k) % L + L) % L];
        y[t] = s;
    }
}

/* The convolution theorem at exactly L points (no padding; L a power of
 * two): DFT both, multiply, inverse DFT, scale by 1/L. */
static void cconv_fft(const double *h, const double *u, long L, double *y, fft_scratch *s)
{
    for (long t = 0; t < L; ++t) {
        s->hr[t] = h[t]; s->hi[t] = 0.0;
        s->ur[t] = u[t]; s->ui[t] = 0.0;
    }
    fft_radix2(s->hr, s->hi, L, -1);
    fft_radix2(s->ur, s->ui, L, -1);
    for (long k = 0; k < L; ++k) {
        const double re = s->hr[k] * s->ur[k] - s->hi[k] * s->ui[k];
        const double im = s->hr[k] * s->ui[k] + s->hi[k] * s->ur[k];
        s->ur[k] = re;
        s->ui[k] = im;
    }
    fft_radix2(s->ur, s->ui, L, +1);
    for (long t = 0; t < L; ++t) y[t] = s->ur[t] / (double)L;
}

int oracle_cconv(const double *h, const double *u, long L, int route, double *y)
{
    if (!h || !u || !y || L < 1) return ORACLE_EBADARG;
    if (route == ROUTE_DIRECT) {
        cconv_direct(h, u, L, y);
        return ORACLE_OK;
    }
    if (route != ROUTE_FFT || !is_pow2(L)) return ORACLE_EBADARG;
    fft_scratch s;
    if (scratch_alloc(&s, L) != ORACLE_OK) {
        scratch_free(&s);
        return ORACLE_ENOMEM;
    }
    cconv_fft(h, u, L, y, &s);
    scratch_free(&s);
    return ORACLE_OK;
}

/* L-point spectrum of each row of h[rows][L] (no padding): bins 0..L/2. */
int oracle_rfft_circ(const double *h, long rows, long L, double *out_re, double *out_im)
{
    if (!h || !out_re || !out_im || rows < 0 || L < 2 || !is_pow2(L)) return ORACLE_EBADARG;
    double *re = malloc(sizeof(double) * L), *im = malloc(sizeof(double) * L);
    if (!re || !im) { free(re); free(im); return ORACLE_ENOMEM; }
    for (long r = 0; r < rows; ++r) {
        for (long t = 0; t < L; ++t) { re[t] = h[r * L + t]; im[t] = 0.0; }
        fft_radix2(re, im, L, -1);
        for (long k = 0; k <= L / 2; ++k) {
            out_re[r * (L / 2 + 1) + k] = re[k];
            out_im[r * (L / 2 + 1) + k] = im[k];
        }
    }
    free(re); free(im);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------ */
/* The order-N Hyena recurrence, 1-D.                                  */
/* ------------------------------------------------------------------ */

typedef struct {
    const double *v, *x, *h, *bias;
    long B, D, L, N;
    int route;
    double *y;
    long s0, step; /* sequences s0, s0 + step, ... (s = b*D + d) */
    int status;
    int circular;  /* 1: circular convolution of length L instead of causal */
} fwd_job;

static void *forward_worker(void *arg)
{
    fwd_job *j = (fwd_job *)arg;
    const long L = j->L, BDL = j->B * j->D * L;
    double *z = malloc(sizeof(double) * L), *c = malloc(sizeof(double) * L);
    fft_scratch s = {0};
    if (!z || !c || (j->route == ROUTE_FFT &&
                     scratch_alloc(&s, j->circular ? L : next_pow2(2 * L)) != ORACLE_OK)) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (long seq = j->s0; seq < j->B * j->D; seq += j->step) {
        const long d = seq % j->D;
        memcpy(z, j->v + seq * L, sizeof(double) * L); /* z_0 = v */
        for (long n = 0; n < j->N; ++n) {
            const double *hn = j->h + (n * j->D + d) * L;
            const double *xn = j->x + n * BDL + seq * L;
            const double bn = j->bias[n * j->D + d];
            if (j->circular) {
                if (j->route == ROUTE_DIRECT) cconv_direct(hn, z, L, c);
                else cconv_fft(hn, z, L, c, &s);
            } else {
                if (j->route == ROUTE_DIRECT) conv_direct(hn, z, L, c);
                else conv_fft(hn, z, L, c, &s);
            }
            /* z_n = x_n * (h_n (*) z_{n-1} + b_n z_{n-1}) */
            for (long t = 0; t < L; ++t) z[t] = xn[t] * (c[t] + bn * z[t]);
        }
        memcpy(j->y + seq * L, z, sizeof(double) * L); /* y = z_N */
    }
    j->status = ORACLE_OK;
done:
    free(z); free(c);
    if (j->route == ROUTE_FFT) scratch_free(&s);
    return NULL;
}

static int forward_any(const double *v, const double *x, const double *h, const double *bias,
                       long B, long D, long L, long N, int route, int nthreads, int circular,
                       double *y);

/* v [B][D][L], x [N][B][D][L], h [N][D][L], bias [N][D] -> y [B][D][L]. */
int oracle_hyena_forward(const double *v, const double *x, const double *h,
                         const double *bias, long B, long D, long L, long N,
                         int route, int nthreads, double *y)
{
    return forward_any(v, x, h, bias, B, D, L, N, route, nthreads, 0, y);
}

/* The same recurrence with circular convolutions of length L (L a power of
 * two for the FFT route). */
int oracle_hyena_forward_circular(const double *v, const double *x, const double *h,
                                  const double *bias, long B, long D, long L, long N,
                                  int route, int nthreads, double *y)
{
    if (route == ROUTE_FFT && !is_pow2(L)) return ORACLE_EBADARG;
    return forward_any(v, x, h, bias, B, D, L, N, route, nthreads, 1, y);
}

static int forward_any(const double *v, const double *x, const double *h, const double *bias,
                       long B, long D, long L, long N, int route, int nthreads, int circular,
                       double *y)
{
    if (!v || !x || !h || !bias || !y || B < 1 || D < 1 || L < 1 || N < 1 ||
        (route != ROUTE_DIRECT && route != ROUTE_FFT))
        return ORACLE_EBADARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * D) nthreads = (int)(B * D);
    fwd_job *jobs = calloc(nthreads, sizeof(fwd_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fwd_job j = {v, x, h, bias, B, D, L, N, route, y, k, nthreads, 0, circular};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, forward_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* ------------------------------------------------------------------ */
/* The backward pass of the 1-D recurrence: the exact adjoint.          */
/* ------------------------------------------------------------------ */
/*
 * The pages give no training formulas; the gradient of a composition is
 * fixed by the chain rule.  With c_n = h_n (*) z_{n-1} + b_n z_{n-1} and
 * z_n = x_n c_n, and g = dL/dz_n flowing back from g = dy at n = N:
 *     dx_n          = g * c_n
 *     e             = g * x_n                       (dL/dc_n)
 *     dh_n[d][s]   += sum_t e[t] z_{n-1}[t - s]     (s = 0..L-1, t >= s)
 *     db_n[d]      += sum_t e[t] z_{n-1}[t]
 *     dz_{n-1}[u]   = sum_{t >= u} h_n[t - u] e[t] + b_n e[u]
 * and dv = dz_0.  dh and db are summed over the batch.
 */

/* Adjoint of the causal convolution with respect to its signal:
 * out[u] = sum_{t=u..L-1} h[t-u] e[t]. */
static void corr_direct(const double *h, const double *e, long L, double *out)
{
    for (long u = 0; u < L; ++u) {
        double s = 0.0;
        for (long t = u; t < L; ++t) s += h[t - u] * e[t];
        out[u] = s;
    }
}

/* Lagged products: out[s] = sum_{t=s..L-1} e[t] z[t-s]. */
static void lagged_direct(const double *e, const double *z, long L, double *out)
{
    for (long s = 0; s < L; ++s) {
        double acc = 0.0;
        for (long t = s; t < L; ++t) acc += e[t] * z[t - s];
        out[s] = acc;
    }
}

/* out[s] = sum_t a[t + s] b[t] for s = 0..L-1 through the DFT of both
 * zero-padded to P >= 2L: IDFT(A conj(B)) / P at s.  Both corr_direct
 * (a = e, b = h) and lagged_direct (a = e, b = z) have this form. */
static void corr_fft(const double *a, const double *b, long L, double *out,
                     fft_scratch *s)
{
    const long P = s->P;
    for (long t = 0; t < P; ++t) {
        s->hr[t] = t < L ? b[t] : 0.0; s->hi[t] = 0.0;
        s->ur[t] = t < L ? a[t] : 0.0; s->ui[t] = 0.0;
    }
    fft_radix2(s->hr, s->hi, P, -1);
    fft_radix2(s->ur, s->ui, P, -1);
    for (long k = 0; k < P; ++k) {
        /* A conj(B) */
        const double re = s->ur[k] * s->hr[k] + s->ui[k] * s->hi[k];
        const double im = s->ui[k] * s->hr[k] - s->ur[k] * s->hi[k];
        s->ur[k] = re;
        s->ui[k] = im;
    }
    fft_radix2(s->ur, s->ui, P, +1);
    for (long t = 0; t < L; ++t) out[t] = s->ur[t] / (double)P;
}

/* Circular counterpart of both sums above (length-L circular convolution,
 * "Handling Boundaries": periodic systems): out[s] = sum_t a[t] b[(t - s)
 * mod L], s = 0..L-1.  With a = e, b = z it is dh; with a = e, b = h the
 * adjoint of the circular convolution with respect to its signal.  Its FFT
 * route is corr_fft with scratch of exactly L points (no padding, so the
 * product of spectra wraps around). */
static void ccorr_direct(const double *a, const double *b, long L, double *out)
{
    for (long s = 0; s < L; ++s) {
        double acc = 0.0;
        for (long t = 0; t < L; ++t) acc += a[t] * b[((t - s) % L + L) % L];
        out[s] = acc;
    }
}

typedef struct {
    const double *v, *x, *h, *bias, *dy;
    long B, D, L, N;
    int route;
    double *dv, *dx, *dh, *dbias;
    long d0, step; /* channels d0, d0 + step, ... (dh, db summed over b here) */
    int status;
    int circular;  /* 1: the recurrence with circular convolutions of length L */
} bwd_job;

static void *backward_worker(void *arg)
{
    bwd_job *j = (bwd_job *)arg;
    const long L = j->L, N = j->N, D = j->D, BDL = j->B * D * L;
    /* z[n] = z_n for n = 0..N-1, c[n] = c_{n+1}; g, e, tmp: length L */
    double *z = malloc(sizeof(double) * N * L), *c = malloc(sizeof(double) * N * L);
    double *g = malloc(sizeof(double) * L), *e = malloc(sizeof(double) * L);
    double *tmp = malloc(sizeof(double) * L);
    fft_scratch s = {0};
    if (!z || !c || !g || !e || !tmp ||
        (j->route == ROUTE_FFT && scratch_alloc(&s, j->circular ? L : next_pow2(2 * L)) != ORACLE_OK)) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (long d = j->d0; d < D; d += j->step) {
        for (long n = 0; n < N; ++n) {
            memset(j->dh + (n * D + d) * L, 0, sizeof(double) * L);
            j->dbias[n * D + d] = 0.0;
        }
        for (long b = 0; b < j->B; ++b) {
            const long seq = b * D + d;
            /* forward, keeping z_{n-1} and c_n */
            memcpy(z, j->v + seq * L, sizeof(double) * L);
            for (long n = 0; n < N; ++n) {
                const double *hn = j->h + (n * D + d) * L;
                const double *xn = j->x + n * BDL + seq * L;
                const double bn = j->bias[n * D + d];
                double *zn = z + n * L, *cn = c + n * L;
                if (j->circular) {
                    if (j->route == ROUTE_DIRECT) cconv_direct(hn, zn, L, cn);
                    else cconv_fft(hn, zn, L, cn, &s);
                } else {
                    if (j->route == ROUTE_DIRECT) conv_direct(hn, zn, L, cn);
                    else conv_fft(hn, zn, L, cn, &s);
                }
                for (long t = 0; t < L; ++t) cn[t] += bn * zn[t];
                if (n + 1 < N)
                    for (long t = 0; t < L; ++t) z[(n + 1) * L + t] = xn[t] * cn[t];
            }
            /* backward */
            memcpy(g, j->dy + seq * L, sizeof(double) * L);
            for (long n = N - 1; n >= 0; --n) {
                const double *hn = j->h + (n * D + d) * L;
                const double *xn = j->x + n * BDL + seq * L;
                const double bn = j->bias[n * D + d];
                const double *zn = z + n * L, *cn = c + n * L;
                double *dxn = j->dx + n * BDL + seq * L;
                double *dhn = j->dh + (n * D + d) * L;
                for (long t = 0; t < L; ++t) {
                    dxn[t] = g[t] * cn[t];
                    e[t] = g[t] * xn[t];
                }
                if (j->route == ROUTE_FFT) corr_fft(e, zn, L, tmp, &s);
                else if (j->circular) ccorr_direct(e, zn, L, tmp);
                else lagged_direct(e, zn, L, tmp);
                for (long t = 0; t < L; ++t) dhn[t] += tmp[t];
                double db = 0.0;
                for (long t = 0; t < L; ++t) db += e[t] * zn[t];
                j->dbias[n * D + d] += db;
                if (j->route == ROUTE_FFT) corr_fft(e, hn, L, tmp, &s);
                else if (j->circular) ccorr_direct(e, hn, L, tmp);
                else corr_direct(hn, e, L, tmp);
                for (long t = 0; t < L; ++t) g[t] = tmp[t] + bn * e[t];
            }
            memcpy(j->dv + seq * L, g, sizeof(double) * L); /* dv = dz_0 */
        }
    }
    j->status = ORACLE_OK;
done:
    free(z); free(c); free(g); free(e); free(tmp);
    if (j->route == ROUTE_FFT) scratch_free(&s);
    return NULL;
}

/* Gradients of a scalar loss with dL/dy = dy [B][D][L]: dv [B][D][L],
 * dx [N][B][D][L], dh [N][D][L] and dbias [N][D] (both summed over the
 * batch).  Inputs as oracle_hyena_forward. */
static int backward_any(const double *v, const double *x, const double *h, const double *bias,
                        const double *dy, long B, long D, long L, long N, int route, int nthreads,
                        int circular, double *dv, double *dx, double *dh, double *dbias);

int oracle_hyena_backward(const double *v, const double *x, const double *h,
                          const double *bias, const double *dy, long B, long D,
                          long L, long N, int route, int nthreads, double *dv,
                          double *dx, double *dh, double *dbias)
{
    return backward_any(v, x, h, bias, dy, B, D, L, N, route, nthreads, 0, dv, dx, dh, dbias);
}

/* The same gradients through the recurrence with circular convolutions of
 * length L (oracle_hyena_forward_circular): dh_n[s] = sum_b sum_t e[t]
 * z_{n-1}[(t - s) mod L], dz_{n-1}[u] = sum_t h_n[(t - u) mod L] e[t] +
 * b_n e[u].  L a power of two for the FFT route. */
int oracle_hyena_backward_circular(const double *v, const double *x, const double *h,
                                   const double *bias, const double *dy, long B, long D,
                                   long L, long N, int route, int nthreads, double *dv,
                                   double *dx, double *dh, double *dbias)
{
    if (route == ROUTE_FFT && !is_pow2(L)) return ORACLE_EBADARG;
    return backward_any(v, x, h, bias, dy, B, D, L, N, route, nthreads, 1, dv, dx, dh, dbias);
}

static int backward_any(const double *v, const double *x, const double *h, const double *bias,
                        const double *dy, long B, long D, long L, long N, int route, int nthreads,
                        int circular, double *dv, double *dx, double *dh, double *dbias)
{
    if (!v || !x || !h || !bias || !dy || !dv || !dx || !dh || !dbias || B < 1 ||
        D < 1 || L < 1 || N < 1 || (route != ROUTE_DIRECT && route != ROUTE_FFT))
        return ORACLE_EBADARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > D) nthreads = (int)D;
    bwd_job *jobs = calloc(nthreads, sizeof(bwd_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        bwd_job j = {v, x, h, bias, dy, B, D, L, N, route, dv, dx, dh, dbias, k, nthreads, 0, circular};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, backward_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* ------------------------------------------------------------------ */
/* 2-D: linear convolution on the grid (Native ND Convolution;         */
/* Handling Boundaries: zero-pad to double the grid).                  */
/* ------------------------------------------------------------------ */

/* The definition: y[p][q] = sum_{i<=p, j<=q} h[i][j] u[p-i][q-j]. */
static void conv2_direct(const double *h, const double *u, long H, long W,
                         double *y)
{
    for (long p = 0; p < H; ++p)
        for (long q = 0; q < W; ++q) {
            double s = 0.0;
            for (long i = 0; i <= p; ++i)
                for (long j = 0; j <= q; ++j)
                    s += h[i * W + j] * u[(p - i) * W + (q - j)];
            y[p * W + q] = s;
        }
}

typedef struct {
    double *hr, *hi, *ur, *ui, *cr, *ci;
    long PH, PW;
} fft2_scratch;

static int scratch2_alloc(fft2_scratch *s, long PH, long PW)
{
    s->PH = PH; s->PW = PW;
    s->hr = malloc(sizeof(double) * PH * PW); s->hi = malloc(sizeof(double) * PH * PW);
    s->ur = malloc(sizeof(double) * PH * PW); s->ui = malloc(sizeof(double) * PH * PW);
    s->cr = malloc(sizeof(double) * PH); s->ci = malloc(sizeof(double) * PH);
    return (s->hr && s->hi && s->ur && s->ui && s->cr && s->ci) ? ORACLE_OK
                                                               : ORACLE_ENOMEM;
}

static void scratch2_free(fft2_scratch *s)
{
    free(s->hr); free(s->hi); free(s->ur); free(s->ui); free(s->cr); free(s->ci);
}

/* 2-D DFT of a PH x PW row-major grid: every row, then every column. */
static void fft2(double *re, double *im, fft2_scratch *s, int sign)
{
    const long PH = s->PH, PW = s->PW;
    for (long y = 0; y < PH; ++y) fft_radix2(re + y * PW, im + y * PW, PW, sign);
    for (long x = 0; x < PW; ++x) {
        for (long y = 0; y < PH; ++y) { s->cr[y] = re[y * PW + x]; s->ci[y] = im[y * PW + x]; }
        fft_radix2(s->cr, s->ci, PH, sign);
        for (long y = 0; y < PH; ++y) { re[y * PW + x] = s->cr[y]; im[y * PW + x] = s->ci[y]; }
    }
}

static void conv2_fft(const double *h, const double *u, long H, long W,
                      double *y, fft2_scratch *s)
{
    const long PH = s->PH, PW = s->PW;
    for (long r = 0; r < PH; ++r)
        for (long q = 0; q < PW; ++q) {
            const int in = r < H && q < W;
            s->hr[r * PW + q] = in ? h[r * W + q] : 0.0; s->hi[r * PW + q] = 0.0;
            s->ur[r * PW + q] = in ? u[r * W + q] : 0.0; s->ui[r * PW + q] = 0.0;
        }
    fft2(s->hr, s->hi, s, -1);
    fft2(s->ur, s->ui, s, -1);
    for (long k = 0; k < PH * PW; ++k) {
        const double re = s->hr[k] * s->ur[k] - s->hi[k] * s->ui[k];
        const double im = s->hr[k] * s->ui[k] + s->hi[k] * s->ur[k];
        s->ur[k] = re;
        s->ui[k] = im;
    }
    fft2(s->ur, s->ui, s, +1);
    for (long r = 0; r < H; ++r)
        for (long q = 0; q < W; ++q)
            y[r * W + q] = s->ur[r * PW + q] / (double)(PH * PW);
}

int oracle_conv2(const double *h, const double *u, long H, long W, int route,
                 double *y)
{
    if (!h || !u || !y || H < 1 || W < 1) return ORACLE_EBADARG;
    if (route == ROUTE_DIRECT) {
        conv2_direct(h, u, H, W, y);
        return ORACLE_OK;
    }
    if (route != ROUTE_FFT) return ORACLE_EBADARG;
    fft2_scratch s;
    if (scratch2_alloc(&s, next_pow2(2 * H), next_pow2(2 * W)) != ORACLE_OK) {
        scratch2_free(&s);
        return ORACLE_ENOMEM;
    }
    conv2_fft(h, u, H, W, y, &s);
    scratch2_free(&s);
    return ORACLE_OK;
}

typedef struct {
    const double *v, *x, *h, *bias;
    long B, C, H, W, N;
    int route;
    double *y;
    long s0, step; /* images s0, s0 + step, ... (s = b*C + c) */
    int status;
} fwd2_job;

static void *forward_2d_worker(void *arg)
{
    fwd2_job *j = (fwd2_job *)arg;
    const long HW = j->H * j->W, BCHW = j->B * j->C * HW;
    double *z = malloc(sizeof(double) * HW), *c = malloc(sizeof(double) * HW);
    fft2_scratch s = {0};
    if (!z || !c || (j->route == ROUTE_FFT &&
                     scratch2_alloc(&s, next_pow2(2 * j->H),
                                    next_pow2(2 * j->W)) != ORACLE_OK)) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (long img = j->s0; img < j->B * j->C; img += j->step) {
        const long ch = img % j->C;
        memcpy(z, j->v + img * HW, sizeof(double) * HW);
        for (long n = 0; n < j->N; ++n) {
            const double *hn = j->h + (n * j->C + ch) * HW;
            const double *xn = j->x + n * BCHW + img * HW;
            const double bn = j->bias[n * j->C + ch];
            if (j->route == ROUTE_DIRECT) conv2_direct(hn, z, j->H, j->W, c);
            else conv2_fft(hn, z, j->H, j->W, c, &s);
            for (long p = 0; p < HW; ++p) z[p] = xn[p] * (c[p] + bn * z[p]);
        }
        memcpy(j->y + img * HW, z, sizeof(double) * HW);
    }
    j->status = ORACLE_OK;
done:
    free(z); free(c);
    if (j->route == ROUTE_FFT) scratch2_free(&s);
    return NULL;
}

/* v [B][C][H][W], x [N][B][C][H][W], h [N][C][H][W], bias [N][C]
 * -> y [B][C][H][W]. */
int oracle_hyena_forward_2d(const double *v, const double *x, const double *h,
                            const double *bias, long B, long C, long H, long W,
                            long N, int route, int nthreads, double *y)
{
    if (!v || !x || !h || !bias || !y || B < 1 || C < 1 || H < 1 || W < 1 ||
        N < 1 || (route != ROUTE_DIRECT && route != ROUTE_FFT))
        return ORACLE_EBADARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * C) nthreads = (int)(B * C);
    fwd2_job *jobs = calloc(nthreads, sizeof(fwd2_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fwd2_job j = {v, x, h, bias, B, C, H, W, N, route, y, k, nthreads, 0};
        jobs[k] = j;
        pthread_create(&tid[k], NULL, forward_2d_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* ------------------------------------------------------------------ */
/* 3-D: linear convolution on a volume (Native ND Convolution;          */
/* Handling Boundaries: zero-pad to double the grid).                  */
/* ------------------------------------------------------------------ */

/* The definition: y[p][q][r] = sum_{i<=p, j<=q, k<=r} h[i][j][k] u[p-i][q-j][r-k]. */
static void conv3_direct(const double *h, const double *u, long Z, long H, long W, double *y)
{
    for (long p = 0; p < Z; ++p)
        for (long q = 0; q < H; ++q)
            for (long r = 0; r < W; ++r) {
                double s = 0.0;
                for (long i = 0; i <= p; ++i)
                    for (long j = 0; j <= q; ++j)
                        for (long k = 0; k <= r; ++k)
                            s += h[(i * H + j) * W + k] * u[((p - i) * H + (q - j)) * W + (r - k)];
                y[(p * H + q) * W + r] = s;
            }
}

/* 3-D DFT of a PZ x PH x PW grid: along x for every (z, y), then along y,
 * then along z, each by the radix-2 routine on a gathered line. */
static int fft3(double *re, double *im, long PZ, long PH, long PW, int sign)
{
    const long n = PZ > PH ? (PZ > PW ? PZ : PW) : (PH > PW ? PH : PW);
    double *lr = malloc(sizeof(double) * n), *li = malloc(sizeof(double) * n);
    if (!lr || !li) { free(lr); free(li); return ORACLE_ENOMEM; }
    for (long z = 0; z < PZ; ++z)
        for (long y = 0; y < PH; ++y) fft_radix2(re + (z * PH + y) * PW, im + (z * PH + y) * PW, PW, sign);
    for (long z = 0; z < PZ; ++z)
        for (long x = 0; x < PW; ++x) {
            for (long y = 0; y < PH; ++y) { lr[y] = re[(z * PH + y) * PW + x]; li[y] = im[(z * PH + y) * PW + x]; }
            fft_radix2(lr, li, PH, sign);
            for (long y = 0; y < PH; ++y) { re[(z * PH + y) * PW + x] = lr[y]; im[(z * PH + y) * PW + x] = li[y]; }
        }
    for (long y = 0; y < PH; ++y)
        for (long x = 0; x < PW; ++x) {
            for (long z = 0; z < PZ; ++z) { lr[z] = re[(z * PH + y) * PW + x]; li[z] = im[(z * PH + y) * PW + x]; }
            fft_radix2(lr, li, PZ, sign);
            for (long z = 0; z < PZ; ++z) { re[(z * PH + y) * PW + x] = lr[z]; im[(z * PH + y) * PW + x] = li[z]; }
        }
    free(lr); free(li);
    return ORACLE_OK;
}

/* The convolution theorem on the grid padded to 2Z x 2H x 2W (powers of two). */
static int conv3_fft(const double *h, const double *u, long Z, long H, long W, double *y)
{
    const long PZ = 2 * Z, PH = 2 * H, PW = 2 * W, P = PZ * PH * PW;
    double *hr = calloc(P, sizeof(double)), *hi = calloc(P, sizeof(double));
    double *ur = calloc(P, sizeof(double)), *ui = calloc(P, sizeof(double));
    int st = ORACLE_ENOMEM;
    if (!hr || !hi || !ur || !ui) goto out;
    for (long z = 0; z < Z; ++z)
        for (long q = 0; q < H; ++q)
            for (long r = 0; r < W; ++r) {
                hr[(z * PH + q) * PW + r] = h[(z * H + q) * W + r];
                ur[(z * PH + q) * PW + r] = u[(z * H + q) * W + r];
            }
    if ((st = fft3(hr, hi, PZ, PH, PW, -1)) != ORACLE_OK) goto out;
    if ((st = fft3(ur, ui, PZ, PH, PW, -1)) != ORACLE_OK) goto out;
    for (long k = 0; k < P; ++k) {
        const double re = hr[k] * ur[k] - hi[k] * ui[k], im = hr[k] * ui[k] + hi[k] * ur[k];
        ur[k] = re;
        ui[k] = im;
    }
    if ((st = fft3(ur, ui, PZ, PH, PW, +1)) != ORACLE_OK) goto out;
    for (long z = 0; z < Z; ++z)
        for (long q = 0; q < H; ++q)
            for (long r = 0; r < W; ++r) y[(z * H + q) * W + r] = ur[(z * PH + q) * PW + r] / (double)P;
out:
    free(hr); free(hi); free(ur); free(ui);
    return st;
}

int oracle_conv3(const double *h, const double *u, long Z, long H, long W, int route, double *y)
{
    if (!h || !u || !y || Z < 1 || H < 1 || W < 1) return ORACLE_EBADARG;
    if (route == ROUTE_DIRECT) {
        conv3_direct(h, u, Z, H, W, y);
        return ORACLE_OK;
    }
    if (route != ROUTE_FFT || !is_pow2(Z) || !is_pow2(H) || !is_pow2(W)) return ORACLE_EBADARG;
    return conv3_fft(h, u, Z, H, W, y);
}

/* v [B][C][Z][H][W], x [N][B][C][Z][H][W], h [N][C][Z][H][W], bias [N][C]
 * -> y [B][C][Z][H][W]: the recurrence with 3-D convolutions (one thread;
 * the 3-D tests are small). */
int oracle_hyena_forward_3d(const double *v, const double *x, const double *h, const double *bias,
                            long B, long C, long Z, long H, long W, long N, int route, double *y)
{
    if (!v || !x || !h || !bias || !y || B < 1 || C < 1 || Z < 1 || H < 1 || W < 1 || N < 1)
        return ORACLE_EBADARG;
    const long V = Z * H * W, BCV = B * C * V;
    double *z = malloc(sizeof(double) * V), *c = malloc(sizeof(double) * V);
    if (!z || !c) { free(z); free(c); return ORACLE_ENOMEM; }
    int st = ORACLE_OK;
    for (long img = 0; img < B * C && st == ORACLE_OK; ++img) {
        const long ch = img % C;
        memcpy(z, v + img * V, sizeof(double) * V);
        for (long n = 0; n < N && st == ORACLE_OK; ++n) {
            const double *hn = h + (n * C + ch) * V, *xn = x + n * BCV + img * V;
            const double bn = bias[n * C + ch];
            st = oracle_conv3(hn, z, Z, H, W, route, c);
            for (long t = 0; t < V; ++t) z[t] = xn[t] * (c[t] + bn * z[t]);
        }
        memcpy(y + img * V, z, sizeof(double) * V);
    }
    free(z); free(c);
    return st;
}

/* ------------------------------------------------------------------ */
/* The backward pass of the 3-D recurrence: the exact adjoint, as in   */
/* 1-D and 2-D, with 3-D correlations.                                  */
/* ------------------------------------------------------------------ */

/* out[a][b][c] = sum_{t >= a, s >= b, u >= c} p[t][s][u] q[t-a][s-b][u-c]:
 * with p = e, q = z it is dh; with p = e, q = h the adjoint of the linear
 * 3-D convolution with respect to its signal.  The definition, O(V^2). */
static void lagged3_direct(const double *p, const double *q, long Z, long H, long W, double *out)
{
    for (long a = 0; a < Z; ++a)
        for (long b = 0; b < H; ++b)
            for (long c = 0; c < W; ++c) {
                double acc = 0.0;
                for (long t = a; t < Z; ++t)
                    for (long s = b; s < H; ++s)
                        for (long u = c; u < W; ++u)
                            acc += p[(t * H + s) * W + u] * q[((t - a) * H + (s - b)) * W + (u - c)];
                out[(a * H + b) * W + c] = acc;
            }
}

/* The same through the DFT of both zero-padded to 2Z x 2H x 2W (powers of
 * two): IDFT(P conj(Q)) / (8 Z H W) at a < Z, b < H, c < W. */
static int lagged3_fft(const double *p, const double *q, long Z, long H, long W, double *out)
{
    const long PZ = 2 * Z, PH = 2 * H, PW = 2 * W, P = PZ * PH * PW;
    double *pr = calloc(P, sizeof(double)), *pi = calloc(P, sizeof(double));
    double *qr = calloc(P, sizeof(double)), *qi = calloc(P, sizeof(double));
    int st = ORACLE_ENOMEM;
    if (!pr || !pi || !qr || !qi) goto out;
    for (long z = 0; z < Z; ++z)
        for (long y = 0; y < H; ++y)
            for (long x = 0; x < W; ++x) {
                pr[(z * PH + y) * PW + x] = p[(z * H + y) * W + x];
                qr[(z * PH + y) * PW + x] = q[(z * H + y) * W + x];
            }
    if ((st = fft3(pr, pi, PZ, PH, PW, -1)) != ORACLE_OK) goto out;
    if ((st = fft3(qr, qi, PZ, PH, PW, -1)) != ORACLE_OK) goto out;
    for (long k = 0; k < P; ++k) {
        const double re = pr[k] * qr[k] + pi[k] * qi[k], im = pi[k] * qr[k] - pr[k] * qi[k];
        pr[k] = re;
        pi[k] = im;
    }
    if ((st = fft3(pr, pi, PZ, PH, PW, +1)) != ORACLE_OK) goto out;
    for (long z = 0; z < Z; ++z)
        for (long y = 0; y < H; ++y)
            for (long x = 0; x < W; ++x) out[(z * H + y) * W + x] = pr[(z * PH + y) * PW + x] / (double)P;
out:
    free(pr); free(pi); free(qr); free(qi);
    return st;
}

/* Gradients of a scalar loss with dL/dy = dy [B][C][Z][H][W] through the
 * 3-D recurrence (oracle_hyena_forward_3d): dv, dx [N][B][C][Z][H][W],
 * dh [N][C][Z][H][W] and dbias [N][C] (both summed over the batch).  With
 * c_n = h_n (*) z_{n-1} + b_n z_{n-1}, z_n = x_n c_n and g = dL/dz_n:
 * dx_n = g c_n, e = g x_n, dh_n += lagged3(e, z_{n-1}), db_n += sum e
 * z_{n-1}, dz_{n-1} = lagged3(e, h_n) + b_n e.  One thread. */
int oracle_hyena_backward_3d(const double *v, const double *x, const double *h, const double *bias,
                             const double *dy, long B, long C, long Z, long H, long W, long N, int route,
                             double *dv, double *dx, double *dh, double *dbias)
{
    if (!v || !x || !h || !bias || !dy || !dv || !dx || !dh || !dbias || B < 1 || C < 1 || Z < 1 || H < 1 ||
        W < 1 || N < 1 || (route != ROUTE_DIRECT && route != ROUTE_FFT))
        return ORACLE_EBADARG;
    if (route == ROUTE_FFT && (!is_pow2(Z) || !is_pow2(H) || !is_pow2(W))) return ORACLE_EBADARG;
    const long V = Z * H * W, BCV = B * C * V;
    double *z = malloc(sizeof(double) * N * V), *c = malloc(sizeof(double) * N * V);
    double *g = malloc(sizeof(double) * V), *e = malloc(sizeof(double) * V), *tmp = malloc(sizeof(double) * V);
    int st = ORACLE_OK;
    if (!z || !c || !g || !e || !tmp) { st = ORACLE_ENOMEM; goto done; }
    memset(dh, 0, sizeof(double) * N * C * V);
    memset(dbias, 0, sizeof(double) * N * C);
    for (long img = 0; img < B * C && st == ORACLE_OK; ++img) {
        const long ch = img % C;
        memcpy(z, v + img * V, sizeof(double) * V);              /* z_0 = v */
        for (long n = 0; n < N && st == ORACLE_OK; ++n) {
            const double *hn = h + (n * C + ch) * V, *xn = x + n * BCV + img * V;
            const double bn = bias[n * C + ch];
            double *zn = z + n * V, *cn = c + n * V;
            st = oracle_conv3(hn, zn, Z, H, W, route, cn);
            for (long t = 0; t < V; ++t) cn[t] += bn * zn[t];
            if (n + 1 < N)
                for (long t = 0; t < V; ++t) z[(n + 1) * V + t] = xn[t] * cn[t];
        }
        memcpy(g, dy + img * V, sizeof(double) * V);
        for (long n = N - 1; n >= 0 && st == ORACLE_OK; --n) {
            const double *hn = h + (n * C + ch) * V, *xn = x + n * BCV + img * V;
            const double bn = bias[n * C + ch];
            const double *zn = z + n * V, *cn = c + n * V;
            double *dxn = dx + n * BCV + img * V, *dhn = dh + (n * C + ch) * V;
            for (long t = 0; t < V; ++t) {
                dxn[t] = g[t] * cn[t];
                e[t] = g[t] * xn[t];
            }
            if (route == ROUTE_DIRECT) lagged3_direct(e, zn, Z, H, W, tmp);
            else st = lagged3_fft(e, zn, Z, H, W, tmp);
            for (long t = 0; t < V; ++t) dhn[t] += tmp[t];
            double db = 0.0;
            for (long t = 0; t < V; ++t) db += e[t] * zn[t];
            dbias[n * C + ch] += db;
            if (route == ROUTE_DIRECT) lagged3_direct(e, hn, Z, H, W, tmp);
            else if (st == ORACLE_OK) st = lagged3_fft(e, hn, Z, H, W, tmp);
            for (long t = 0; t < V; ++t) g[t] = tmp[t] + bn * e[t];
        }
        memcpy(dv + img * V, g, sizeof(double) * V);             /* dv = dz_0 */
    }
done:
    free(z); free(c); free(g); free(e); free(tmp);
    return st;
}

/* ------------------------------------------------------------------ */
/* Circular convolution on 2-D grids and 3-D volumes (Handling          */
/* Boundaries: circular convolutions for periodic physical systems; a   */
/* 2-D grid is a volume with Z = 1).                                    */
/* ------------------------------------------------------------------ */

/* The definition: y[p][q][r] = sum_{i,j,k} h[i][j][k]
 * u[(p-i) mod Z][(q-j) mod H][(r-k) mod W]. */
static void cconv3_direct(const double *h, const double *u, long Z, long H, long W, double *y)
{
    for (long p = 0; p < Z; ++p)
        for (long q = 0; q < H; ++q)
            for (long r = 0; r < W; ++r) {
                double s = 0.0;
                for (long i = 0; i < Z; ++i)
                    for (long j = 0; j < H; ++j)
                        for (long k = 0; k < W; ++k) {
                            const long a = (p - i + Z) % Z, b = (q - j + H) % H, c = (r - k + W) % W;
                            s += h[(i * H + j) * W + k] * u[(a * H + b) * W + c];
                        }
                y[(p * H + q) * W + r] = s;
            }
}

/* The convolution theorem on the Z x H x W grid itself (no padding; powers
 * of two): 3-D DFT of both, multiply, inverse, scale by 1/(Z H W). */
static int cconv3_fft(const double *h, const double *u, long Z, long H, long W, double *y)
{
    const long P = Z * H * W;
    double *hr = malloc(sizeof(double) * P), *hi = calloc(P, sizeof(double));
    double *ur = malloc(sizeof(double) * P), *ui = calloc(P, sizeof(double));
    int st = ORACLE_ENOMEM;
    if (!hr || !hi || !ur || !ui) goto out;
    memcpy(hr, h, sizeof(double) * P);
    memcpy(ur, u, sizeof(double) * P);
    if ((st = fft3(hr, hi, Z, H, W, -1)) != ORACLE_OK) goto out;
    if ((st = fft3(ur, ui, Z, H, W, -1)) != ORACLE_OK) goto out;
    for (long k = 0; k < P; ++k) {
        const double re = hr[k] * ur[k] - hi[k] * ui[k], im = hr[k] * ui[k] + hi[k] * ur[k];
        ur[k] = re;
        ui[k] = im;
    }
    if ((st = fft3(ur, ui, Z, H, W, +1)) != ORACLE_OK) goto out;
    for (long k = 0; k < P; ++k) y[k] = ur[k] / (double)P;
out:
    free(hr); free(hi); free(ur); free(ui);
    return st;
}

int oracle_cconv3(const double *h, const double *u, long Z, long H, long W, int route, double *y)
{
    if (!h || !u || !y || Z < 1 || H < 1 || W < 1) return ORACLE_EBADARG;
    if (route == ROUTE_DIRECT) {
        cconv3_direct(h, u, Z, H, W, y);
        return ORACLE_OK;
    }
    if (route != ROUTE_FFT || !is_pow2(Z) || !is_pow2(H) || !is_pow2(W)) return ORACLE_EBADARG;
    return cconv3_fft(h, u, Z, H, W, y);
}

/* v [B][C][Z][H][W], x [N][B][C][Z][H][W], h [N][C][Z][H][W], bias [N][C]
 * -> y [B][C][Z][H][W]: the recurrence with circular convolutions on the
 * grid (Z = 1 for 2-D), one thread. */
int oracle_hyena_forward_circular_nd(const double *v, const double *x, const double *h,
                                     const double *bias, long B, long C, long Z, long H, long W,
                                     long N, int route, double *y)
{
    if (!v || !x || !h || !bias || !y || B < 1 || C < 1 || Z < 1 || H < 1 || W < 1 || N < 1)
        return ORACLE_EBADARG;
    const long V = Z * H * W, BCV = B * C * V;
    double *z = malloc(sizeof(double) * V), *c = malloc(sizeof(double) * V);
    if (!z || !c) { free(z); free(c); return ORACLE_ENOMEM; }
    int st = ORACLE_OK;
    for (long img = 0; img < B * C && st == ORACLE_OK; ++img) {
        const long ch = img % C;
        memcpy(z, v + img * V, sizeof(double) * V);
        for (long n = 0; n < N && st == ORACLE_OK; ++n) {
            const double *hn = h + (n * C + ch) * V, *xn = x + n * BCV + img * V;
            const double bn = bias[n * C + ch];
            st = oracle_cconv3(hn, z, Z, H, W, route, c);
            for (long t = 0; t < V; ++t) z[t] = xn[t] * (c[t] + bn * z[t]);
        }
        memcpy(y + img * V, z, sizeof(double) * V);
    }
    free(z); free(c);
    return st;
}

/* ------------------------------------------------------------------ */
/* Backward of the circular 3-D recurrence (oracle_hyena_forward_       */
/* circular_nd): the chain rule with both sums wrapping around.         */
/* ------------------------------------------------------------------ */

/* out[a][b][c] = sum_{t,s,u} p[t][s][u] q[(t-a) mod Z][(s-b) mod H][(u-c)
 * mod W].  With p = e, q = z it is dh; with p = e, q = h the adjoint of the
 * circular 3-D convolution with respect to its signal.  The definition. */
static void ccorr3_direct(const double *p, const double *q, long Z, long H, long W, double *out)
{
    for (long a = 0; a < Z; ++a)
        for (long b = 0; b < H; ++b)
            for (long c = 0; c < W; ++c) {
                double acc = 0.0;
                for (long t = 0; t < Z; ++t)
                    for (long s = 0; s < H; ++s)
                        for (long u = 0; u < W; ++u)
                            acc += p[(t * H + s) * W + u] *
                                   q[(((t - a + Z) % Z) * H + (s - b + H) % H) * W + (u - c + W) % W];
                out[(a * H + b) * W + c] = acc;
            }
}

/* The same through the DFT on the Z x H x W grid itself (powers of two, no
 * padding, so the product wraps): IDFT(P conj(Q)) / (Z H W). */
static int ccorr3_fft(const double *p, const double *q, long Z, long H, long W, double *out)
{
    const long P = Z * H * W;
    double *pr = malloc(sizeof(double) * P), *pi = calloc(P, sizeof(double));
    double *qr = malloc(sizeof(double) * P), *qi = calloc(P, sizeof(double));
    int st = ORACLE_ENOMEM;
    if (!pr || !pi || !qr || !qi) goto out;
    memcpy(pr, p, sizeof(double) * P);
    memcpy(qr, q, sizeof(double) * P);
    if ((st = fft3(pr, pi, Z, H, W, -1)) != ORACLE_OK) goto out;
    if ((st = fft3(qr, qi, Z, H, W, -1)) != ORACLE_OK) goto out;
    for (long k = 0; k < P; ++k) {
        const double re = pr[k] * qr[k] + pi[k] * qi[k], im = pi[k] * qr[k] - pr[k] * qi[k];
        pr[k] = re;
        pi[k] = im;
    }
    if ((st = fft3(pr, pi, Z, H, W, +1)) != ORACLE_OK) goto out;
    for (long k = 0; k < P; ++k) out[k] = pr[k] / (double)P;
out:
    free(pr); free(pi); free(qr); free(qi);
    return st;
}

/* Gradients of a scalar loss with dL/dy = dy [B][C][Z][H][W] through the
 * circular 3-D recurrence: dv, dx [N][B][C][Z][H][W], dh [N][C][Z][H][W]
 * and dbias [N][C] (both summed over the batch).  With c_n = h_n (*) z_{n-1}
 * + b_n z_{n-1} (circular), z_n = x_n c_n and g = dL/dz_n: dx_n = g c_n,
 * e = g x_n, dh_n += ccorr3(e, z_{n-1}), db_n += sum e z_{n-1},
 * dz_{n-1} = ccorr3(e, h_n) + b_n e.  One thread. */
int oracle_hyena_backward_circular_3d(const double *v, const double *x, const double *h,
                                      const double *bias, const double *dy, long B, long C, long Z, long H,
                                      long W, long N, int route, double *dv, double *dx, double *dh,
                                      double *dbias)
{
    if (!v || !x || !h || !bias || !dy || !dv || !dx || !dh || !dbias || B < 1 || C < 1 || Z < 1 || H < 1 ||
        W < 1 || N < 1 || (route != ROUTE_DIRECT && route != ROUTE_FFT))
        return ORACLE_EBADARG;
    if (route == ROUTE_FFT && (!is_pow2(Z) || !is_pow2(H) || !is_pow2(W))) return ORACLE_EBADARG;
    const long V = Z * H * W, BCV = B * C * V;
    double *z = malloc(sizeof(double) * N * V), *c = malloc(sizeof(double) * N * V);
    double *g = malloc(sizeof(double) * V), *e = malloc(sizeof(double) * V), *tmp = malloc(sizeof(double) * V);
    int st = ORACLE_OK;
    if (!z || !c || !g || !e || !tmp) { st = ORACLE_ENOMEM; goto done; }
    memset(dh, 0, sizeof(double) * N * C * V);
    memset(dbias, 0, sizeof(double) * N * C);
    for (long img = 0; img < B * C && st == ORACLE_OK; ++img) {
        const long ch = img % C;
        memcpy(z, v + img * V, sizeof(double) * V);              /* z_0 = v */
        for (long n = 0; n < N && st == ORACLE_OK; ++n) {
            const double *hn = h + (n * C + ch) * V, *xn = x + n * BCV + img * V;
            const double bn = bias[n * C + ch];
            double *zn = z + n * V, *cn = c + n * V;
            st = oracle_cconv3(hn, zn, Z, H, W, route, cn);
            for (long t = 0; t < V; ++t) cn[t] += bn * zn[t];
            if (n + 1 < N)
                for (long t = 0; t < V; ++t) z[(n + 1) * V + t] = xn[t] * cn[t];
        }
        memcpy(g, dy + img * V, sizeof(double) * V);
        for (long n = N - 1; n >= 0 && st == ORACLE_OK; --n) {
            const double *hn = h + (n * C + ch) * V, *xn = x + n * BCV + img * V;
            const double bn = bias[n * C + ch];
            const double *zn = z + n * V, *cn = c + n * V;
            double *dxn = dx + n * BCV + img * V, *dhn = dh + (n * C + ch) * V;
            for (long t = 0; t < V; ++t) {
                dxn[t] = g[t] * cn[t];
                e[t] = g[t] * xn[t];
            }
            if (route == ROUTE_DIRECT) ccorr3_direct(e, zn, Z, H, W, tmp);
            else st = ccorr3_fft(e, zn, Z, H, W, tmp);
            for (long t = 0; t < V; ++t) dhn[t] += tmp[t];
            double db = 0.0;
            for (long t = 0; t < V; ++t) db += e[t] * zn[t];
            dbias[n * C + ch] += db;
            if (route == ROUTE_DIRECT) ccorr3_direct(e, hn, Z, H, W, tmp);
            else if (st == ORACLE_OK) st = ccorr3_fft(e, hn, Z, H, W, tmp);
            for (long t = 0; t < V; ++t) g[t] = tmp[t] + bn * e[t];
        }
        memcpy(dv + img * V, g, sizeof(double) * V);             /* dv = dz_0 */
    }
done:
    free(z); free(c); free(g); free(e); free(tmp);
    return st;
}

/* ------------------------------------------------------------------ */
/* Backward of the 2-D recurrence (the chain rule, as in 1-D, with the  */
/* 2-D linear convolution of Native ND Convolution / Handling           */
/* Boundaries):                                                         */
/*     dx_n = g c_n,  e = g x_n,                                        */
/*     dh_n[a][b] += sum_{t,s} e[t][s] z_{n-1}[t-a][s-b],               */
/*     db_n += sum e z_{n-1} = dh_n[0][0],                              */
/*     g <- sum_{t>=u, s>=w} h_n[t-u][s-w] e[t][s] + b_n e,  dv = g.    */
/* ------------------------------------------------------------------ */

/* Adjoint of the 2-D convolution with respect to its signal:
 * out[u][w] = sum_{t>=u, s>=w} h[t-u][s-w] e[t][s]. */
static void corr2_direct(const double *h, const double *e, long H, long W, double *out)
{
    for (long u = 0; u < H; ++u)
        for (long w = 0; w < W; ++w) {
            double acc = 0.0;
            for (long t = u; t < H; ++t)
                for (long s = w; s < W; ++s) acc += h[(t - u) * W + (s - w)] * e[t * W + s];
            out[u * W + w] = acc;
        }
}

/* Lagged products: out[a][b] = sum_{t>=a, s>=b} e[t][s] z[t-a][s-b]. */
static void lagged2_direct(const double *e, const double *z, long H, long W, double *out)
{
    for (long a = 0; a < H; ++a)
        for (long b = 0; b < W; ++b) {
            double acc = 0.0;
            for (long t = a; t < H; ++t)
                for (long s = b; s < W; ++s) acc += e[t * W + s] * z[(t - a) * W + (s - b)];
            out[a * W + b] = acc;
        }
}

/* out[a][b] = sum_{t,s} p[t+a][s+b] q[t][s] for a < H, b < W: the 2-D DFT
 * of both zero-padded to PH x PW >= 2H x 2W, IDFT(P conj(Q)) / (PH PW).
 * corr2_direct (p = e, q = h) and lagged2_direct (p = e, q = z) both have
 * this form. */
static void corr2_fft(const double *p, const double *q, long H, long W, double *out, fft2_scratch *s)
{
    const long PH = s->PH, PW = s->PW;
    for (long r = 0; r < PH; ++r)
        for (long c = 0; c < PW; ++c) {
            const int in = r < H && c < W;
            s->ur[r * PW + c] = in ? p[r * W + c] : 0.0; s->ui[r * PW + c] = 0.0;
            s->hr[r * PW + c] = in ? q[r * W + c] : 0.0; s->hi[r * PW + c] = 0.0;
        }
    fft2(s->ur, s->ui, s, -1);
    fft2(s->hr, s->hi, s, -1);
    for (long k = 0; k < PH * PW; ++k) {
        const double re = s->ur[k] * s->hr[k] + s->ui[k] * s->hi[k];
        const double im = s->ui[k] * s->hr[k] - s->ur[k] * s->hi[k];
        s->ur[k] = re;
        s->ui[k] = im;
    }
    fft2(s->ur, s->ui, s, +1);
    for (long r = 0; r < H; ++r)
        for (long c = 0; c < W; ++c) out[r * W + c] = s->ur[r * PW + c] / (double)(PH * PW);
}

/* Circular counterpart of both 2-D sums (periodic boundaries, "Handling
 * Boundaries"): out[a][b] = sum_{t,s} p[t][s] q[(t - a) mod H][(s - b) mod
 * W].  With p = e, q = z it is dh; with p = e, q = h the adjoint of the
 * circular convolution with respect to its signal.  Its FFT route is
 * corr2_fft on an H x W scratch (no padding, so the product wraps). */
static void ccorr2_direct(const double *p, const double *q, long H, long W, double *out)
{
    for (long a = 0; a < H; ++a)
        for (long b = 0; b < W; ++b) {
            double acc = 0.0;
            for (long t = 0; t < H; ++t)
                for (long s = 0; s < W; ++s)
                    acc += p[t * W + s] * q[((t - a + H) % H) * W + (s - b + W) % W];
            out[a * W + b] = acc;
        }
}

typedef struct {
    const double *v, *x, *h, *bias, *dy;
    long B, C, H, W, N;
    int route;
    double *dv, *dx, *dh, *dbias;
    long c0, step; /* channels c0, c0 + step, ... (dh, db summed over b here) */
    int status;
    int circular;  /* 1: circular convolutions on the H x W grid itself */
} bwd2_job;

static void *backward_2d_worker(void *arg)
{
    bwd2_job *j = (bwd2_job *)arg;
    const long HW = j->H * j->W, N = j->N, C = j->C, BCHW = j->B * C * HW;
    double *z = malloc(sizeof(double) * N * HW), *c = malloc(sizeof(double) * N * HW);
    double *g = malloc(sizeof(double) * HW), *e = malloc(sizeof(double) * HW);
    double *tmp = malloc(sizeof(double) * HW);
    fft2_scratch s = {0};
    if (!z || !c || !g || !e || !tmp ||
        (j->route == ROUTE_FFT &&
         scratch2_alloc(&s, j->circular ? j->H : next_pow2(2 * j->H),
                        j->circular ? j->W : next_pow2(2 * j->W)) != ORACLE_OK)) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (long ch = j->c0; ch < C; ch += j->step) {
        for (long n = 0; n < N; ++n) {
            memset(j->dh + (n * C + ch) * HW, 0, sizeof(double) * HW);
            j->dbias[n * C + ch] = 0.0;
        }
        for (long b = 0; b < j->B; ++b) {
            const long img = b * C + ch;
            /* forward, keeping z_{n-1} and c_n */
            memcpy(z, j->v + img * HW, sizeof(double) * HW);
            for (long n = 0; n < N; ++n) {
                const double *hn = j->h + (n * C + ch) * HW, *xn = j->x + n * BCHW + img * HW;
                const double bn = j->bias[n * C + ch];
                double *zn = z + n * HW, *cn = c + n * HW;
                if (j->circular) {
                    if (j->route == ROUTE_DIRECT) cconv3_direct(hn, zn, 1, j->H, j->W, cn);
                    else conv2_fft(hn, zn, j->H, j->W, cn, &s);   /* H x W scratch: wraps */
                } else if (j->route == ROUTE_DIRECT) {
                    conv2_direct(hn, zn, j->H, j->W, cn);
                } else {
                    conv2_fft(hn, zn, j->H, j->W, cn, &s);
                }
                for (long t = 0; t < HW; ++t) cn[t] += bn * zn[t];
                if (n + 1 < N)
                    for (long t = 0; t < HW; ++t) z[(n + 1) * HW + t] = xn[t] * cn[t];
            }
            /* backward */
            memcpy(g, j->dy + img * HW, sizeof(double) * HW);
            for (long n = N - 1; n >= 0; --n) {
                const double *hn = j->h + (n * C + ch) * HW, *xn = j->x + n * BCHW + img * HW;
                const double bn = j->bias[n * C + ch];
                const double *zn = z + n * HW, *cn = c + n * HW;
                double *dxn = j->dx + n * BCHW + img * HW, *dhn = j->dh + (n * C + ch) * HW;
                for (long t = 0; t < HW; ++t) {
                    dxn[t] = g[t] * cn[t];
                    e[t] = g[t] * xn[t];
                }
                if (j->route == ROUTE_FFT) corr2_fft(e, zn, j->H, j->W, tmp, &s);
                else if (j->circular) ccorr2_direct(e, zn, j->H, j->W, tmp);
                else lagged2_direct(e, zn, j->H, j->W, tmp);
                for (long t = 0; t < HW; ++t) dhn[t] += tmp[t];
                double db = 0.0;
                for (long t = 0; t < HW; ++t) db += e[t] * zn[t];
                j->dbias[n * C + ch] += db;
                if (j->route == ROUTE_FFT) corr2_fft(e, hn, j->H, j->W, tmp, &s);
                else if (j->circular) ccorr2_direct(e, hn, j->H, j->W, tmp);
                else corr2_direct(hn, e, j->H, j->W, tmp);
                for (long t = 0; t < HW; ++t) g[t] = tmp[t] + bn * e[t];
            }
            memcpy(j->dv + img * HW, g, sizeof(double) * HW);
        }
    }
    j->status = ORACLE_OK;
done:
    free(z); free(c); free(g); free(e); free(tmp);
    if (j->route == ROUTE_FFT) scratch2_free(&s);
    return NULL;
}

/* Gradients of a scalar loss with dL/dy = dy [B][C][H][W] through the 2-D
 * recurrence: dv [B][C][H][W], dx [N][B][C][H][W], dh [N][C][H][W] and
 * dbias [N][C] (both summed over the batch). */
static int backward_2d_any(const double *v, const double *x, const double *h, const double *bias,
                           const double *dy, long B, long C, long H, long W, long N, int route,
                           int nthreads, int circular, double *dv, double *dx, double *dh, double *dbias);

int oracle_hyena_backward_2d(const double *v, const double *x, const double *h, const double *bias,
                             const double *dy, long B, long C, long H, long W, long N, int route,
                             int nthreads, double *dv, double *dx, double *dh, double *dbias)
{
    return backward_2d_any(v, x, h, bias, dy, B, C, H, W, N, route, nthreads, 0, dv, dx, dh, dbias);
}

/* The same gradients through the 2-D recurrence with circular convolutions
 * on the H x W grid itself (oracle_hyena_forward_circular_nd with Z = 1):
 * dh_n[a][b] = sum_b' sum_{t,s} e[t][s] z_{n-1}[(t - a) mod H][(s - b) mod W],
 * dz_{n-1}[u][w] = sum_{t,s} h_n[(t - u) mod H][(s - w) mod W] e[t][s] +
 * b_n e[u][w].  H, W powers of two for the FFT route. */
int oracle_hyena_backward_circular_2d(const double *v, const double *x, const double *h,
                                      const double *bias, const double *dy, long B, long C, long H,
                                      long W, long N, int route, int nthreads, double *dv, double *dx,
                                      double *dh, double *dbias)
{
    if (route == ROUTE_FFT && (!is_pow2(H) || !is_pow2(W))) return ORACLE_EBADARG;
    return backward_2d_any(v, x, h, bias, dy, B, C, H, W, N, route, nthreads, 1, dv, dx, dh, dbias);
}

static int backward_2d_any(const double *v, const double *x, const double *h, const double *bias,
                           const double *dy, long B, long C, long H, long W, long N, int route,
                           int nthreads, int circular, double *dv, double *dx, double *dh, double *dbias)
{
    if (!v || !x || !h || !bias || !dy || !dv || !dx || !dh || !dbias || B < 1 || C < 1 || H < 1 ||
        W < 1 || N < 1 || (route != ROUTE_DIRECT && route != ROUTE_FFT))
        return ORACLE_EBADARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > C) nthreads = (int)C;
    bwd2_job *jobs = calloc(nthreads, sizeof(bwd2_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        bwd2_job jb = {v, x, h, bias, dy, B, C, H, W, N, route, dv, dx, dh, dbias, k, nthreads, 0, circular};
        jobs[k] = jb;
        pthread_create(&tid[k], NULL, backward_2d_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* ------------------------------------------------------------------ */
/* Implicit 3-D filters: the filter network of the 1-D and 2-D forms on */
/* positional features of a volume (Native ND Convolution: a global     */
/* filter on an L1 x ... x LN grid, produced by the implicit filter MLP */
/* from the position).  Features [tz, ty, tx, (sin, cos)(2 pi k tz),    */
/* (sin, cos)(2 pi k ty), (sin, cos)(2 pi k tx)], k = 1..K, t = i / n   */
/* per axis; window exp(-alpha_c (iz + iy + ix) / decay_div), the       */
/* product of the three axis windows.                                   */
/* ------------------------------------------------------------------ */

typedef struct {
    const double *W1, *W2, *W3, *Wout, *alpha;
    int N, C, Z, H, W, n_bands, width;
    double decay_div;
    double *h;
    long p0, p1; /* flattened volume positions handled by this worker */
    int status;
} fg3_job;

static void *filter_gen_3d_worker(void *arg)
{
    fg3_job *j = (fg3_job *)arg;
    const int K = j->n_bands, n_in = 3 + 6 * K, n_out = j->N * j->C;
    const long V = (long)j->Z * j->H * j->W;
    double *phi = malloc(sizeof(double) * n_in);
    double *a1 = malloc(sizeof(double) * j->width), *a2 = malloc(sizeof(double) * j->width);
    double *a3 = malloc(sizeof(double) * j->width), *o = malloc(sizeof(double) * n_out);
    if (!phi || !a1 || !a2 || !a3 || !o) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (long p = j->p0; p < j->p1; ++p) {
        const long iz = p / ((long)j->H * j->W), iy = (p / j->W) % j->H, ix = p % j->W;
        const double t[3] = {(double)iz / j->Z, (double)iy / j->H, (double)ix / j->W};
        for (int a = 0; a < 3; ++a) {
            phi[a] = t[a];
            for (int k = 1; k <= K; ++k) {
                phi[3 + 2 * K * a + 2 * (k - 1)] = sin(2.0 * ORACLE_PI * k * t[a]);
                phi[3 + 2 * K * a + 2 * (k - 1) + 1] = cos(2.0 * ORACLE_PI * k * t[a]);
            }
        }
        ffn(j->W1, j->W2, j->W3, j->Wout, n_in, j->width, n_out, phi, a1, a2, a3, o);
        for (int n = 0; n < j->N; ++n)
            for (int c = 0; c < j->C; ++c) {
                const double window = exp(-j->alpha[c] * (double)(iz + iy + ix) / j->decay_div);
                j->h[((long)n * j->C + c) * V + p] = o[n * j->C + c] * window;
            }
    }
    j->status = ORACLE_OK;
done:
    free(phi); free(a1); free(a2); free(a3); free(o);
    return NULL;
}

/* h[N][C][Z][H][W] from the FFN weights (W1 [width][3+6K]) and alpha[C]. */
int oracle_filter_gen_3d(const double *W1, const double *W2, const double *W3, const double *Wout,
                         const double *alpha, int N, int C, int Z, int H, int W, int n_bands, int width,
                         double decay_div, int nthreads, double *h)
{
    if (!W1 || !W2 || !W3 || !Wout || !alpha || !h || N < 1 || C < 1 || Z < 1 || H < 1 || W < 1 ||
        n_bands < 0 || width < 1 || !(decay_div > 0.0))
        return ORACLE_EBADARG;
    const long V = (long)Z * H * W;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > V) nthreads = (int)V;
    fg3_job *jobs = calloc(nthreads, sizeof(fg3_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fg3_job jb = {W1, W2, W3, Wout, alpha, N, C, Z, H, W, n_bands, width, decay_div, h,
                      V * k / nthreads, V * (k + 1) / nthreads, 0};
        jobs[k] = jb;
        pthread_create(&tid[k], NULL, filter_gen_3d_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}

/* Input-dependent 3-D filters: the FiLM-modulated sine layers of
 * oracle_filter_gen_film on the 3-D features of oracle_filter_gen_3d,
 * h[B][N][C][Z][H][W]; the window is the separable exponential decay of
 * oracle_filter_gen_3d (gaussian = 0, win = alpha) or the Gaussian
 * exp(-(tz^2 + ty^2 + tx^2) / (2 sigma_c^2)) (gaussian = 1, win = sigma). */
typedef struct {
    const double *W1, *W2, *W3, *Wout, *omega, *gamma, *beta, *win;
    int gaussian, B, N, C, Z, H, W, n_bands, width;
    double decay_div;
    double *h;
    long p0, p1;
    int status;
} fgf3_job;

static void *filter_gen_film_3d_worker(void *arg)
{
    fgf3_job *j = (fgf3_job *)arg;
    const int K = j->n_bands, n_in = 3 + 6 * K, w = j->width, n_out = j->N * j->C;
    const long V = (long)j->Z * j->H * j->W;
    double *phi = malloc(sizeof(double) * n_in);
    double *a1 = malloc(sizeof(double) * w), *a2 = malloc(sizeof(double) * w);
    double *a3 = malloc(sizeof(double) * w), *o = malloc(sizeof(double) * n_out);
    if (!phi || !a1 || !a2 || !a3 || !o) {
        j->status = ORACLE_ENOMEM;
        goto done;
    }
    for (int b = 0; b < j->B; ++b) {
        const double *g = j->gamma + (long)b * 3 * w, *be = j->beta + (long)b * 3 * w;
        for (long p = j->p0; p < j->p1; ++p) {
            const long iz = p / ((long)j->H * j->W), iy = (p / j->W) % j->H, ix = p % j->W;
            const double t[3] = {(double)iz / j->Z, (double)iy / j->H, (double)ix / j->W};
            for (int a = 0; a < 3; ++a) {
                phi[a] = t[a];
                for (int k = 1; k <= K; ++k) {
                    phi[3 + 2 * K * a + 2 * (k - 1)] = sin(2.0 * ORACLE_PI * k * t[a]);
                    phi[3 + 2 * K * a + 2 * (k - 1) + 1] = cos(2.0 * ORACLE_PI * k * t[a]);
                }
            }
            matvec(j->W1, w, n_in, phi, a1);
            film_sin(a1, w, j->omega, g, be);
            matvec(j->W2, w, w, a1, a2);
            film_sin(a2, w, j->omega + w, g + w, be + w);
            matvec(j->W3, w, w, a2, a3);
            film_sin(a3, w, j->omega + 2 * w, g + 2 * w, be + 2 * w);
            matvec(j->Wout, n_out, w, a3, o);
            for (int n = 0; n < j->N; ++n)
                for (int c = 0; c < j->C; ++c) {
                    const double s = j->win[c];
                    const double window =
                        j->gaussian ? exp(-(t[0] * t[0] + t[1] * t[1] + t[2] * t[2]) / (2.0 * s * s))
                                    : exp(-s * (double)(iz + iy + ix) / j->decay_div);
                    j->h[(((long)b * j->N + n) * j->C + c) * V + p] = o[n * j->C + c] * window;
                }
        }
    }
    j->status = ORACLE_OK;
done:
    free(phi); free(a1); free(a2); free(a3); free(o);
    return NULL;
}

int oracle_filter_gen_film_3d(const double *W1, const double *W2, const double *W3, const double *Wout,
                              const double *omega, const double *gamma, const double *beta, const double *win,
                              int gaussian, int B, int N, int C, int Z, int H, int W, int n_bands, int width,
                              double decay_div, int nthreads, double *h)
{
    if (!W1 || !W2 || !W3 || !Wout || !omega || !gamma || !beta || !win || !h || B < 1 || N < 1 || C < 1 ||
        Z < 1 || H < 1 || W < 1 || n_bands < 0 || width < 1 || !(decay_div > 0.0))
        return ORACLE_EBADARG;
    const long V = (long)Z * H * W;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > V) nthreads = (int)V;
    fgf3_job *jobs = calloc(nthreads, sizeof(fgf3_job));
    pthread_t *tid = calloc(nthreads, sizeof(pthread_t));
    if (!jobs || !tid) { free(jobs); free(tid); return ORACLE_ENOMEM; }
    for (int k = 0; k < nthreads; ++k) {
        fgf3_job jb = {W1, W2, W3, Wout, omega, gamma, beta, win, gaussian, B, N, C, Z, H, W, n_bands, width,
                       decay_div, h, V * k / nthreads, V * (k + 1) / nthreads, 0};
        jobs[k] = jb;
        pthread_create(&tid[k], NULL, filter_gen_film_3d_worker, &jobs[k]);
    }
    int st = ORACLE_OK;
    for (int k = 0; k < nthreads; ++k) {
        pthread_join(tid[k], NULL);
        if (jobs[k].status != ORACLE_OK) st = jobs[k].status;
    }
    free(jobs); free(tid);
    return st;
}
