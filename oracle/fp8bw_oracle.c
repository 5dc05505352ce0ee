/*
 * fp8bw_oracle.c -- plain, slow CPU reference ("oracle") for the blockwise-FP8
 * training linear layer of the Puro-2B recipe.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may call this code. It shares nothing with the
 * CUDA path (no header, table, helper or constant generator).
 *
 * Build: gcc -std=c11 -O2 -fno-fast-math -ffp-contract=off -fPIC -shared
 *        (x86-64 SSE arithmetic: every float operation below is one IEEE-754
 *        binary32 operation rounded to nearest-even, with no FMA contraction).
 *
 * Sources and readings are listed in fp8bw_oracle.h. Each function below says
 * which passage it follows.
 *
 * Parity pins: every function here is pinned by the tests under tests/ that
 * are marked "not gpu" (torch's float8_e4m3fn conversion for the codec,
 * hand-worked groups, exact lossless-quantisation products, exact rational
 * brute force at 4x4x256, and an fp64 dequantise-then-matmul cross-check).
 */
#include "fp8bw_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* E4M3 format (OCP 8-bit floating point, E4M3 variant).                     */
/* The report names the format only as "E4M3" (arxiv-wiki summary, Approach  */
/* item (4); paperlayer.ai summary, Appendix C production settings). Its     */
/* definition: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no  */
/* infinities; S.1111.111 is NaN; exponent field 0 is subnormal m * 2^-9.     */
/* ------------------------------------------------------------------------ */

double orc_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int ef = (code >> 3) & 0xF;
    int mf = code & 0x7;
    double mag;
    if (ef == 0xF && mf == 0x7)
        return NAN;
    if (ef == 0)
        mag = ldexp((double)mf, -9);                  /* subnormal: m * 2^-9 */
    else
        mag = ldexp(1.0 + mf / 8.0, ef - 7);          /* (1 + m/8) * 2^(e-7) */
    return sign ? -mag : mag;
}

/* Round a non-negative double to an integer, ties to even. */
static double round_half_even(double v)
{
    double fl = floor(v);
    double frac = v - fl;                 /* exact: v has few significant bits */
    if (frac > 0.5)
        return fl + 1.0;
    if (frac < 0.5)
        return fl;
    return (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0;
}

/* fp32 -> E4M3, round to nearest even, saturating finite values to +-448.
 * The pages leave rounding and overflow open; this takes the reading
 * "round-to-nearest-even, clamp to the largest finite value". */
uint8_t orc_e4m3_encode(float t)
{
    uint8_t sign = signbit(t) ? 0x80 : 0x00;
    double a = fabs((double)t);
    int e;
    double m;

    if (isnan(t))
        return (uint8_t)(sign | 0x7F);
    if (a >= 448.0)                       /* largest finite E4M3 is 1.75 * 2^8 */
        return (uint8_t)(sign | 0x7E);

    /* Exponent of a: a = f * 2^e with f in [0.5, 1). */
    if (a == 0.0)
        return sign;
    (void)frexp(a, &e);
    e -= 1;                               /* now a in [2^e, 2^(e+1)) */

    if (e < -6) {
        /* Subnormal range: the grid is k * 2^-9, k = 0..8 (k = 8 is 2^-6, the
         * smallest normal, whose code 0x08 is also just k). */
        m = round_half_even(ldexp(a, 9));
        return (uint8_t)(sign | (uint8_t)m);
    }

    /* Normal range: a = (8 + f) * 2^(e-3), f = 0..7. */
    m = round_half_even(ldexp(a, 3 - e)); /* in [8, 16] */
    if (m == 16.0) {                      /* rounded up into the next binade */
        m = 8.0;
        e += 1;
    }
    /* a < 448 keeps e <= 8 and the code below 0x7E-or-equal. */
    return (uint8_t)(sign | (uint8_t)((e + 7) << 3) | (uint8_t)(m - 8.0));
}

/* Element-wise encode of an array (same conversion as orc_e4m3_encode). */
void orc_e4m3_encode_array(const float* t, int64_t count, uint8_t* out)
{
    int64_t i;
    for (i = 0; i < count; ++i)
        out[i] = orc_e4m3_encode(t[i]);
}

/* Integer value of an E4M3 code in units of 2^-9 (every finite E4M3 number is
 * an integer multiple of 2^-9; |value| <= 448 * 512 = 229376). The 256 values
 * are taken from orc_e4m3_decode once and kept in a table. */
static int32_t g_units[256];
static pthread_once_t g_units_once = PTHREAD_ONCE_INIT;

static void build_units(void)
{
    int c;
    for (c = 0; c < 256; ++c) {
        double v = orc_e4m3_decode((uint8_t)c);
        g_units[c] = isnan(v) ? 0 : (int32_t)ldexp(v, 9);
    }
}

static int32_t e4m3_units(uint8_t code)
{
    return g_units[code];
}

/* ------------------------------------------------------------------------ */
/* bf16 helpers                                                              */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round a double to bf16 (8 significant bits), nearest-even, one rounding. */
uint16_t orc_bf16_round(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0x0000;
    double a = fabs(v);
    int e;
    double m;
    float f;
    uint32_t u;

    if (isnan(v))
        return 0x7FC0;
    if (a == 0.0)
        return sign;
    (void)frexp(a, &e);
    e -= 1;                               /* a in [2^e, 2^(e+1)) */
    if (e < -126)
        e = -126;                         /* subnormal spacing 2^-133 */
    m = round_half_even(ldexp(a, 7 - e)); /* quantum 2^(e-7) */
    a = ldexp(m, e - 7);
    if (a > 3.3895313892515355e38)        /* above the largest finite bf16 */
        return (uint16_t)(sign | 0x7F80);
    f = (float)a;                         /* exact: a has <= 8 significant bits */
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (uint16_t)(u >> 16));
}

/* ------------------------------------------------------------------------ */
/* Group scale.  Report: "block scale" per 1-D group of 128 (activations) or */
/* per 128x128 block (weights) -- arxiv-wiki summary, Approach item (4). The */
/* formula is the max-abs reading: the group's amax is mapped onto 448, the  */
/* largest finite E4M3 magnitude.                                            */
/* ------------------------------------------------------------------------ */

void orc_group_scale(float amax, float* qscale, float* s)
{
    float q = 448.0f / amax;              /* one binary32 division, RNE */
    if (amax == 0.0f || !isfinite(q)) {   /* all-zero (or vanishing) group */
        *qscale = 1.0f;
        *s = 1.0f;
        return;
    }
    *qscale = q;
    *s = amax / 448.0f;                   /* dequantisation scale */
}

/* Power-of-two variant (the form the B200 tensor cores apply in hardware,
 * UE8M0 scale factors; the pages leave the scale form open -- the arxiv-wiki
 * summary's developer notes only say the grouping and scaling follow the
 * DeepSeek-V3 approach). s = 2^E with E the smallest integer such that
 * 448 * 2^E >= amax, clamped to [-127, 127]; qscale = 2^-E. amax == 0 or a
 * non-finite amax gives qscale = s = 1. The test 448 * 2^E >= amax is exact
 * in binary64. */
void orc_group_scale_pow2(float amax, float* qscale, float* s)
{
    int e;
    if (amax == 0.0f || !isfinite(amax)) {
        *qscale = 1.0f;
        *s = 1.0f;
        return;
    }
    /* start near log2(amax / 448) and step to the smallest valid E */
    (void)frexp((double)amax / 448.0, &e);
    while (ldexp(448.0, e) < (double)amax)
        ++e;
    while (ldexp(448.0, e - 1) >= (double)amax)
        --e;
    if (e < -127)
        e = -127;
    if (e > 127)
        e = 127;
    *qscale = (float)ldexp(1.0, -e);      /* exact: a power of two in range */
    *s = (float)ldexp(1.0, e);            /* 2^-127 is a binary32 subnormal */
}

/* Encode one element of a group: t = x * qscale in binary32, then E4M3. */
static uint8_t encode_elem(uint16_t xb, float qscale)
{
    float t = orc_bf16_to_float(xb) * qscale;
    return orc_e4m3_encode(t);
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

/* Row-wise 1x128 activation quantiser: groups run along the columns (the
 * contraction dimension of the GEMM that consumes the codes). */
typedef void (*scale_fn)(float, float*, float*);

static int quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                            uint8_t* q, float* s, scale_fn scale)
{
    int64_t r, g, c, ngroups;
    if (!x || !q || !s || rows < 0 || cols < 0)
        return -1;
    ngroups = ceil_div(cols, 128);
    for (r = 0; r < rows; ++r) {
        for (g = 0; g < ngroups; ++g) {
            int64_t c0 = g * 128, c1 = c0 + 128 < cols ? c0 + 128 : cols;
            float amax = 0.0f, qscale, sc;
            for (c = c0; c < c1; ++c) {
                float a = fabsf(orc_bf16_to_float(x[r * cols + c]));
                if (a > amax)
                    amax = a;
            }
            scale(amax, &qscale, &sc);
            for (c = c0; c < c1; ++c)
                q[r * cols + c] = encode_elem(x[r * cols + c], qscale);
            s[g * rows + r] = sc;
        }
    }
    return 0;
}

/* Column-wise 128x1 quantiser: groups run along the rows (the token dimension,
 * which is the contraction dimension of the weight-gradient GEMM -- paperlayer.ai
 * summary, Appendix C, "FP8 implementation pipeline"). Codes are written
 * transposed: q_t[col][row]. */
static int quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                            uint8_t* q_t, float* s_t, scale_fn scale)
{
    int64_t r, g, c, ngroups;
    if (!x || !q_t || !s_t || rows < 0 || cols < 0)
        return -1;
    ngroups = ceil_div(rows, 128);
    for (c = 0; c < cols; ++c) {
        for (g = 0; g < ngroups; ++g) {
            int64_t r0 = g * 128, r1 = r0 + 128 < rows ? r0 + 128 : rows;
            float amax = 0.0f, qscale, sc;
            for (r = r0; r < r1; ++r) {
                float a = fabsf(orc_bf16_to_float(x[r * cols + c]));
                if (a > amax)
                    amax = a;
            }
            scale(amax, &qscale, &sc);
            for (r = r0; r < r1; ++r)
                q_t[c * rows + r] = encode_elem(x[r * cols + c], qscale);
            s_t[g * cols + c] = sc;
        }
    }
    return 0;
}

/* Weight quantiser, one scale per 128x128 block (arxiv-wiki summary, Approach
 * item (4)). q_t, when not NULL, receives the same codes transposed. */
static int quantize_weight_block(const uint16_t* w, int64_t n, int64_t k,
                                 uint8_t* q, float* s, uint8_t* q_t,
                                 scale_fn scale)
{
    int64_t nb, kb, i, j, nblk_n, nblk_k;
    if (!w || !q || !s || n < 0 || k < 0)
        return -1;
    nblk_n = ceil_div(n, 128);
    nblk_k = ceil_div(k, 128);
    for (nb = 0; nb < nblk_n; ++nb) {
        for (kb = 0; kb < nblk_k; ++kb) {
            int64_t i0 = nb * 128, i1 = i0 + 128 < n ? i0 + 128 : n;
            int64_t j0 = kb * 128, j1 = j0 + 128 < k ? j0 + 128 : k;
            float amax = 0.0f, qscale, sc;
            for (i = i0; i < i1; ++i)
                for (j = j0; j < j1; ++j) {
                    float a = fabsf(orc_bf16_to_float(w[i * k + j]));
                    if (a > amax)
                        amax = a;
                }
            scale(amax, &qscale, &sc);
            for (i = i0; i < i1; ++i)
                for (j = j0; j < j1; ++j) {
                    uint8_t code = encode_elem(w[i * k + j], qscale);
                    q[i * k + j] = code;
                    if (q_t)
                        q_t[j * n + i] = code;
                }
            s[nb * nblk_k + kb] = sc;
        }
    }
    return 0;
}

int orc_quantize_rowwise(const uint16_t* x, int64_t rows, int64_t cols,
                         uint8_t* q, float* s)
{
    return quantize_rowwise(x, rows, cols, q, s, orc_group_scale);
}

int orc_quantize_colwise(const uint16_t* x, int64_t rows, int64_t cols,
                         uint8_t* q_t, float* s_t)
{
    return quantize_colwise(x, rows, cols, q_t, s_t, orc_group_scale);
}

int orc_quantize_weight_block(const uint16_t* w, int64_t n, int64_t k,
                              uint8_t* q, float* s, uint8_t* q_t)
{
    return quantize_weight_block(w, n, k, q, s, q_t, orc_group_scale);
}

int orc_quantize_rowwise_pow2(const uint16_t* x, int64_t rows, int64_t cols,
                              uint8_t* q, float* s)
{
    return quantize_rowwise(x, rows, cols, q, s, orc_group_scale_pow2);
}

int orc_quantize_colwise_pow2(const uint16_t* x, int64_t rows, int64_t cols,
                              uint8_t* q_t, float* s_t)
{
    return quantize_colwise(x, rows, cols, q_t, s_t, orc_group_scale_pow2);
}

int orc_quantize_weight_block_pow2(const uint16_t* w, int64_t n, int64_t k,
                                   uint8_t* q, float* s, uint8_t* q_t)
{
    return quantize_weight_block(w, n, k, q, s, q_t, orc_group_scale_pow2);
}

/* ------------------------------------------------------------------------ */
/* GEMMs.  paperlayer.ai summary, Appendix C, "FP8 implementation pipeline": */
/* the E4M3 linear-layer GEMMs are forward propagation, data-gradient and    */
/* weight-gradient. With Y = X W^T (W stored [out, in]):                      */
/*   fprop  Y[m][n]  = sum_c sX[c][m]  * sW[n/128][c]  * P_c,                 */
/*          P_c = sum_{k in c} qX[m][k] * qW[n][k]                            */
/*   dgrad  dX[m][k] = sum_c sdY[c][m] * sW[c][k/128]  * P_c,                 */
/*          P_c = sum_{n in c} qdY[m][n] * qW[n][k]                           */
/*   wgrad  dW[n][k] = sum_c sdYt[c][n] * sXt[c][k]    * P_c,                 */
/*          P_c = sum_{m in c} qdYt[n][m] * qXt[k][m]                         */
/* where q means the decoded E4M3 value and c runs over 128-long chunks of    */
/* the contraction dimension. P_c is exact (int64 in units of 2^-18), the     */
/* scale product is exact in fp64, and the chunks are summed in fp64.         */
/* bound = sum over the contraction of |a*b| with a, b dequantised.           */
/* ------------------------------------------------------------------------ */

enum { ROLE_FPROP = 0, ROLE_DGRAD = 1, ROLE_WGRAD = 2 };

typedef struct {
    int role;
    const uint8_t* qa;
    const float* sa;
    const uint8_t* qb;
    const float* sb;
    int64_t m, n, k;          /* the layer's own M (tokens), N (out), K (in) */
} gemm_args;

static void fprop_elem(const gemm_args* g, int64_t mi, int64_t ni,
                       double* acc, double* bound)
{
    int64_t K = g->k, M = g->m, nkb = ceil_div(K, 128), c, kk;
    double y = 0.0, b = 0.0;
    for (c = 0; c < nkb; ++c) {
        int64_t k0 = c * 128, k1 = k0 + 128 < K ? k0 + 128 : K;
        int64_t p = 0, pabs = 0;
        double scale;
        for (kk = k0; kk < k1; ++kk) {
            int64_t prod = (int64_t)e4m3_units(g->qa[mi * K + kk]) *
                           (int64_t)e4m3_units(g->qb[ni * K + kk]);
            p += prod;
            pabs += prod < 0 ? -prod : prod;
        }
        scale = (double)g->sa[c * M + mi] * (double)g->sb[(ni / 128) * nkb + c];
        y += scale * ldexp((double)p, -18);
        b += scale * ldexp((double)pabs, -18);
    }
    *acc = y;
    if (bound)
        *bound = b;
}

static void dgrad_elem(const gemm_args* g, int64_t mi, int64_t ki,
                       double* acc, double* bound)
{
    int64_t K = g->k, M = g->m, N = g->n;
    int64_t nnb = ceil_div(N, 128), nkb = ceil_div(K, 128), c, nn;
    double y = 0.0, b = 0.0;
    (void)nnb;
    for (c = 0; c < nnb; ++c) {
        int64_t n0 = c * 128, n1 = n0 + 128 < N ? n0 + 128 : N;
        int64_t p = 0, pabs = 0;
        double scale;
        for (nn = n0; nn < n1; ++nn) {
            int64_t prod = (int64_t)e4m3_units(g->qa[mi * N + nn]) *
                           (int64_t)e4m3_units(g->qb[nn * K + ki]);
            p += prod;
            pabs += prod < 0 ? -prod : prod;
        }
        scale = (double)g->sa[c * M + mi] * (double)g->sb[c * nkb + ki / 128];
        y += scale * ldexp((double)p, -18);
        b += scale * ldexp((double)pabs, -18);
    }
    *acc = y;
    if (bound)
        *bound = b;
}

static void wgrad_elem(const gemm_args* g, int64_t ni, int64_t ki,
                       double* acc, double* bound)
{
    int64_t K = g->k, M = g->m, N = g->n, nmb = ceil_div(M, 128), c, mm;
    double y = 0.0, b = 0.0;
    for (c = 0; c < nmb; ++c) {
        int64_t m0 = c * 128, m1 = m0 + 128 < M ? m0 + 128 : M;
        int64_t p = 0, pabs = 0;
        double scale;
        for (mm = m0; mm < m1; ++mm) {
            int64_t prod = (int64_t)e4m3_units(g->qa[ni * M + mm]) *
                           (int64_t)e4m3_units(g->qb[ki * M + mm]);
            p += prod;
            pabs += prod < 0 ? -prod : prod;
        }
        scale = (double)g->sa[c * N + ni] * (double)g->sb[c * K + ki];
        y += scale * ldexp((double)p, -18);
        b += scale * ldexp((double)pabs, -18);
    }
    *acc = y;
    if (bound)
        *bound = b;
}

static void gemm_elem(const gemm_args* g, int64_t i, int64_t j, double* acc,
                      double* bound)
{
    if (g->role == ROLE_FPROP)
        fprop_elem(g, i, j, acc, bound);
    else if (g->role == ROLE_DGRAD)
        dgrad_elem(g, i, j, acc, bound);
    else
        wgrad_elem(g, i, j, acc, bound);
}

/* Output shape of each role. */
static void out_shape(const gemm_args* g, int64_t* rows, int64_t* cols)
{
    if (g->role == ROLE_FPROP) {
        *rows = g->m;
        *cols = g->n;
    } else if (g->role == ROLE_DGRAD) {
        *rows = g->m;
        *cols = g->k;
    } else {
        *rows = g->n;
        *cols = g->k;
    }
}

/* Work split for threads: either whole output rows or a list of points. */
typedef struct {
    const gemm_args* g;
    const int64_t* pi;        /* NULL: full output */
    const int64_t* pj;
    int64_t begin, end;       /* rows (full) or point indices */
    double* acc;
    double* bound;
} gemm_work;

static void* gemm_worker(void* arg)
{
    gemm_work* w = (gemm_work*)arg;
    int64_t rows, cols, t, j;
    out_shape(w->g, &rows, &cols);
    (void)rows;
    for (t = w->begin; t < w->end; ++t) {
        if (w->pi) {
            gemm_elem(w->g, w->pi[t], w->pj[t], &w->acc[t],
                      w->bound ? &w->bound[t] : NULL);
        } else {
            for (j = 0; j < cols; ++j)
                gemm_elem(w->g, t, j, &w->acc[t * cols + j],
                          w->bound ? &w->bound[t * cols + j] : NULL);
        }
    }
    return NULL;
}

static int run_gemm(const gemm_args* g, const int64_t* pi, const int64_t* pj,
                    int64_t count, double* acc, double* bound, int nthreads)
{
    gemm_work* work;
    pthread_t* tids;
    char* started;
    int t;
    pthread_once(&g_units_once, build_units);
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > 256)
        nthreads = 256;
    if ((int64_t)nthreads > count)
        nthreads = count > 0 ? (int)count : 1;
    work = (gemm_work*)calloc((size_t)nthreads, sizeof *work);
    tids = (pthread_t*)calloc((size_t)nthreads, sizeof *tids);
    started = (char*)calloc((size_t)nthreads, 1);
    if (!work || !tids || !started) {
        free(work);
        free(tids);
        free(started);
        return -1;
    }
    for (t = 0; t < nthreads; ++t) {
        work[t].g = g;
        work[t].pi = pi;
        work[t].pj = pj;
        work[t].begin = count * t / nthreads;
        work[t].end = count * (t + 1) / nthreads;
        work[t].acc = acc;
        work[t].bound = bound;
    }
    for (t = 1; t < nthreads; ++t)
        started[t] = pthread_create(&tids[t], NULL, gemm_worker, &work[t]) == 0;
    gemm_worker(&work[0]);
    for (t = 1; t < nthreads; ++t) {
        if (started[t])
            pthread_join(tids[t], NULL);
        else
            gemm_worker(&work[t]);      /* thread could not start: run inline */
    }
    free(work);
    free(tids);
    free(started);
    return 0;
}

static int gemm_full(int role, const uint8_t* qa, const float* sa,
                     const uint8_t* qb, const float* sb, int64_t m, int64_t n,
                     int64_t k, double* acc, double* bound, int nthreads)
{
    gemm_args g;
    int64_t rows, cols;
    if (!qa || !sa || !qb || !sb || !acc || m < 0 || n < 0 || k < 0)
        return -1;
    g.role = role;
    g.qa = qa;
    g.sa = sa;
    g.qb = qb;
    g.sb = sb;
    g.m = m;
    g.n = n;
    g.k = k;
    out_shape(&g, &rows, &cols);
    return run_gemm(&g, NULL, NULL, rows, acc, bound, nthreads);
}

static int gemm_points(int role, const uint8_t* qa, const float* sa,
                       const uint8_t* qb, const float* sb, int64_t m,
                       int64_t n, int64_t k, const int64_t* pi,
                       const int64_t* pj, int64_t npts, double* acc,
                       double* bound, int nthreads)
{
    gemm_args g;
    int64_t rows, cols, p;
    if (!qa || !sa || !qb || !sb || !acc || !pi || !pj || m < 0 || n < 0 ||
        k < 0 || npts < 0)
        return -1;
    g.role = role;
    g.qa = qa;
    g.sa = sa;
    g.qb = qb;
    g.sb = sb;
    g.m = m;
    g.n = n;
    g.k = k;
    out_shape(&g, &rows, &cols);
    for (p = 0; p < npts; ++p)
        if (pi[p] < 0 || pi[p] >= rows || pj[p] < 0 || pj[p] >= cols)
            return -1;
    return run_gemm(&g, pi, pj, npts, acc, bound, nthreads);
}

int orc_gemm_fprop(const uint8_t* qx, const float* sx, const uint8_t* qw,
                   const float* sw, int64_t m, int64_t n, int64_t k,
                   double* acc, double* bound, int nthreads)
{
    return gemm_full(ROLE_FPROP, qx, sx, qw, sw, m, n, k, acc, bound, nthreads);
}

int orc_gemm_dgrad(const uint8_t* qdy, const float* sdy, const uint8_t* qw,
                   const float* sw, int64_t m, int64_t n, int64_t k,
                   double* acc, double* bound, int nthreads)
{
    return gemm_full(ROLE_DGRAD, qdy, sdy, qw, sw, m, n, k, acc, bound,
                     nthreads);
}

int orc_gemm_wgrad(const uint8_t* qdy_t, const float* sdy_t,
                   const uint8_t* qx_t, const float* sx_t, int64_t m,
                   int64_t n, int64_t k, double* acc, double* bound,
                   int nthreads)
{
    return gemm_full(ROLE_WGRAD, qdy_t, sdy_t, qx_t, sx_t, m, n, k, acc, bound,
                     nthreads);
}

int orc_gemm_fprop_points(const uint8_t* qx, const float* sx, const uint8_t* qw,
                          const float* sw, int64_t m, int64_t n, int64_t k,
                          const int64_t* pi, const int64_t* pj, int64_t npts,
                          double* acc, double* bound, int nthreads)
{
    return gemm_points(ROLE_FPROP, qx, sx, qw, sw, m, n, k, pi, pj, npts, acc,
                       bound, nthreads);
}

int orc_gemm_dgrad_points(const uint8_t* qdy, const float* sdy,
                          const uint8_t* qw, const float* sw, int64_t m,
                          int64_t n, int64_t k, const int64_t* pi,
                          const int64_t* pj, int64_t npts, double* acc,
                          double* bound, int nthreads)
{
    return gemm_points(ROLE_DGRAD, qdy, sdy, qw, sw, m, n, k, pi, pj, npts,
                       acc, bound, nthreads);
}

int orc_gemm_wgrad_points(const uint8_t* qdy_t, const float* sdy_t,
                          const uint8_t* qx_t, const float* sx_t, int64_t m,
                          int64_t n, int64_t k, const int64_t* pi,
                          const int64_t* pj, int64_t npts, double* acc,
                          double* bound, int nthreads)
{
    return gemm_points(ROLE_WGRAD, qdy_t, sdy_t, qx_t, sx_t, m, n, k, pi, pj,
                       npts, acc, bound, nthreads);
}
