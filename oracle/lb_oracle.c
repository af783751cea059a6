/*
 * Oracle for the LittleBit factorised binary linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file or the library built from it: only the tests, the package
 * smoke check and the CPU-baseline leg of the benchmark do.  It shares no
 * code, header or constant with the CUDA library.
 *
 * What it computes (plain definitions, fp64, no blocking or fusion):
 *
 *   "Samsung LittleBit: A 13B LLM Under 1 GB" (explainx.ai), "How it works",
 *   section 1: W is approximated by the product of two thin matrices U and V,
 *   and at inference only their signs (+1 / -1) are used.  Section 2: learned
 *   FP16 scale vectors along the rows, the columns and the latent dimension.
 *   Section 3: a second, residual branch is added to the first.
 *
 *   Plain reading of those three statements, for one input row x (length in):
 *     u_j   = g_j * x_j                       column scale      (j < in)
 *     t_k   = sum_j s(V_jk) * u_j             binary contraction (k < r)
 *     t'_k  = l_k * t_k                       latent scale
 *     z_i   = h_i * sum_k s(U_ik) * t'_k      binary contraction + row scale
 *     y_i   = z_i(primary) + z_i(residual)
 *   with s(v) = -1 if v < 0 and +1 otherwise (so sign(0) = +1, and a NaN
 *   latent counts as +1).
 *
 * Packed sign format (the reading adopted for "signs, one bit per entry"):
 *   bit (e % 32) of word (e / 32) of a packed row is 1 exactly when latent
 *   element e of that row is < 0; bits past the end of a row are 0.
 *   V (in x r) is packed along `in` for every latent column k: Vp[k][in/32].
 *   U (out x r) is packed along r for every output row i:     Up[i][r/32].
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <stdlib.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Sign of packed element e of one packed row: +1.0 or -1.0. */
static double packed_sign(const uint32_t *row, int64_t e)
{
    uint32_t bit = (row[e >> 5] >> (uint32_t)(e & 31)) & 1u;
    return bit ? -1.0 : 1.0;
}

int lbo_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void lbo_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Pack the signs of an fp32 latent matrix (rows x cols, row stride ld).
 *   axis == 1: every row is packed along its columns -> packed[rows][ld_words]
 *   axis == 0: every column is packed along the rows -> packed[cols][ld_words]
 * Returns 0, or -1 on bad arguments.
 */
int lbo_pack(const float *latent, int64_t rows, int64_t cols, int64_t ld,
             int axis, uint32_t *packed, int64_t ld_words)
{
    if (!latent || !packed || rows < 0 || cols < 0 || ld < cols) return -1;
    if (axis == 1) {
        if (ld_words * 32 < cols) return -1;
#pragma omp parallel for schedule(static)
        for (int64_t i = 0; i < rows; ++i) {
            for (int64_t w = 0; w < ld_words; ++w) {
                uint32_t word = 0;
                for (int b = 0; b < 32; ++b) {
                    int64_t c = w * 32 + b;
                    if (c < cols && latent[i * ld + c] < 0.0f) word |= 1u << b;
                }
                packed[i * ld_words + w] = word;
            }
        }
        return 0;
    }
    if (axis == 0) {
        if (ld_words * 32 < rows) return -1;
        /* one task per group of 32 latent rows: it owns word w of every column */
#pragma omp parallel for schedule(static)
        for (int64_t w = 0; w < ld_words; ++w) {
            for (int64_t c = 0; c < cols; ++c) packed[c * ld_words + w] = 0u;
            for (int b = 0; b < 32; ++b) {
                int64_t i = w * 32 + b;
                if (i >= rows) break;
                for (int64_t c = 0; c < cols; ++c)
                    if (latent[i * ld + c] < 0.0f) packed[c * ld_words + w] |= 1u << b;
            }
        }
        return 0;
    }
    return -1;
}

/*
 * Forward of the factorised binary layer for M input rows.
 *   x      : M x in (fp64, row-major)
 *   Vp[b]  : r rows of ldv words, bits along `in`   (branch b)
 *   Up[b]  : out rows of ldu words, bits along r    (branch b)
 *   h[b]   : out, g[b] : in, l[b] : r                (fp64 copies of the FP16 scales)
 *   rows   : optional list of n_rows output rows to evaluate (NULL = all rows)
 *   y      : M x n_rows (or M x out when rows == NULL), overwritten
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int lbo_forward(const double *x, int64_t M, int64_t in, int64_t out, int64_t r,
                int nb, const uint32_t *const *Vp, int64_t ldv,
                const uint32_t *const *Up, int64_t ldu,
                const double *const *h, const double *const *g,
                const double *const *l, const int64_t *rows, int64_t n_rows,
                double *y)
{
    if (!x || !y || M < 0 || in <= 0 || out <= 0 || r <= 0 || nb < 1) return -1;
    if (ldv * 32 < in || ldu * 32 < r) return -1;
    int64_t ny = rows ? n_rows : out;
    if (rows) {
        if (n_rows < 0) return -1;
        for (int64_t q = 0; q < n_rows; ++q)
            if (rows[q] < 0 || rows[q] >= out) return -1;
    }
    double *u = (double *)malloc(sizeof(double) * (size_t)in);
    double *tp = (double *)malloc(sizeof(double) * (size_t)r);
    if (!u || !tp) { free(u); free(tp); return -1; }

    for (int64_t m = 0; m < M; ++m) {
        double *ym = y + m * ny;
        for (int64_t q = 0; q < ny; ++q) ym[q] = 0.0;
        for (int b = 0; b < nb; ++b) {
            /* column scale */
            for (int64_t j = 0; j < in; ++j) u[j] = g[b][j] * x[m * in + j];
            /* first contraction, then latent scale */
#pragma omp parallel for schedule(static)
            for (int64_t k = 0; k < r; ++k) {
                const uint32_t *vrow = Vp[b] + k * ldv;
                double t = 0.0;
                for (int64_t j = 0; j < in; ++j) t += packed_sign(vrow, j) * u[j];
                tp[k] = l[b][k] * t;
            }
            /* second contraction, then row scale; branches are summed */
#pragma omp parallel for schedule(static)
            for (int64_t q = 0; q < ny; ++q) {
                int64_t i = rows ? rows[q] : q;
                const uint32_t *urow = Up[b] + i * ldu;
                double z = 0.0;
                for (int64_t k = 0; k < r; ++k) z += packed_sign(urow, k) * tp[k];
                ym[q] += h[b][i] * z;
            }
        }
    }
    free(u);
    free(tp);
    return 0;
}

/*
 * Bit-serial variant of the forward ("The XOR claim" on the same page: when
 * both operands are signs, a multiply becomes an XOR plus a popcount).  The
 * activations are not signs, so this variant first quantises each vector to
 * B-bit fixed point in a code whose B bit-planes are themselves signs:
 *
 *   Q_B(v[0..n)): A = max|v_j| (fp32), D = 2^e with e the smallest integer
 *   (e >= -100) such that A <= (2^B - 1) * D; q_j = 2*floor(v_j / (2D)) + 1,
 *   an odd integer in [-(2^B - 1), 2^B - 1], so that |D*q_j - v_j| <= D.
 *   Every odd q in that range is sum_p 2^p sigma_p with sigma_p in {-1, +1}
 *   (sigma_p = 2*bit_p((q + 2^B - 1)/2) - 1).
 *
 * so that sum_j s_j q_j = sum_p 2^p sum_j s_j sigma_jp, a sum of sign-times-
 * sign products.  This oracle takes the definition as written: the integer
 * dot products sum_j s_j q_j directly (the popcount identity is what the GPU
 * side uses and what the tests check it against).  Decisions that choose an
 * integer code are taken in fp32, as the kernel takes them:
 *
 *   u_j  = fp32(g_j * x_j)                         (exact)
 *   (D1, q) = Q_B(u);     T_k = sum_j s(V_jk) q_j  (exact integer)
 *   t'_k = fp32(l_k * fp32(D1 * T_k))
 *   (D2, q') = Q_B(t');   Z_i = sum_k s(U_ik) q'_k (exact integer)
 *   y_i += h_i * D2 * Z_i                          (fp64, summed over branches)
 */
static float xor_scale(const float *v, int64_t n, int B)
{
    float A = 0.0f;
    for (int64_t j = 0; j < n; ++j) {
        float a = fabsf(v[j]);
        if (a > A) A = a;
    }
    const float top = (float)((1L << B) - 1);
    int e = -100;
    /* the smallest e with A <= top * 2^e (exact products of powers of two) */
    if (A > top * ldexpf(1.0f, e)) {
        int ea;
        frexpf(A, &ea);            /* A < 2^ea */
        e = ea - B - 1;
        if (e < -100) e = -100;
        while (A > top * ldexpf(1.0f, e)) ++e;
        while (e > -100 && A <= top * ldexpf(1.0f, e - 1)) --e;
    }
    return ldexpf(1.0f, e);
}

static int64_t xor_code(float v, float D)
{
    return 2 * (int64_t)floorf(v / (2.0f * D)) + 1;
}

int lbo_forward_xor(const double *x, int64_t M, int64_t in, int64_t out, int64_t r,
                    int nb, int B, const uint32_t *const *Vp, int64_t ldv,
                    const uint32_t *const *Up, int64_t ldu,
                    const double *const *h, const double *const *g,
                    const double *const *l, double *y)
{
    if (!x || !y || M < 0 || in <= 0 || out <= 0 || r <= 0 || nb < 1) return -1;
    if (B < 1 || B > 24 || ldv * 32 < in || ldu * 32 < r) return -1;
    float *u = (float *)malloc(sizeof(float) * (size_t)in);
    float *tp = (float *)malloc(sizeof(float) * (size_t)r);
    int64_t *q = (int64_t *)malloc(sizeof(int64_t) * (size_t)in);
    int64_t *q2 = (int64_t *)malloc(sizeof(int64_t) * (size_t)r);
    if (!u || !tp || !q || !q2) { free(u); free(tp); free(q); free(q2); return -1; }
    for (int64_t m = 0; m < M; ++m) {
        double *ym = y + m * out;
        for (int64_t i = 0; i < out; ++i) ym[i] = 0.0;
        for (int b = 0; b < nb; ++b) {
            for (int64_t j = 0; j < in; ++j) u[j] = (float)g[b][j] * (float)x[m * in + j];
            const float D1 = xor_scale(u, in, B);
            for (int64_t j = 0; j < in; ++j) q[j] = xor_code(u[j], D1);
#pragma omp parallel for schedule(static)
            for (int64_t k = 0; k < r; ++k) {
                const uint32_t *vrow = Vp[b] + k * ldv;
                int64_t T = 0;
                for (int64_t j = 0; j < in; ++j)
                    T += (((vrow[j >> 5] >> (uint32_t)(j & 31)) & 1u) ? -q[j] : q[j]);
                const float DT = D1 * (float)T;
                tp[k] = (float)l[b][k] * DT;
            }
            const float D2 = xor_scale(tp, r, B);
            for (int64_t k = 0; k < r; ++k) q2[k] = xor_code(tp[k], D2);
#pragma omp parallel for schedule(static)
            for (int64_t i = 0; i < out; ++i) {
                const uint32_t *urow = Up[b] + i * ldu;
                int64_t Z = 0;
                for (int64_t k = 0; k < r; ++k)
                    Z += (((urow[k >> 5] >> (uint32_t)(k & 31)) & 1u) ? -q2[k] : q2[k]);
                ym[i] += h[b][i] * (double)D2 * (double)Z;
            }
        }
    }
    free(u); free(tp); free(q); free(q2);
    return 0;
}

/* The quantiser alone (for the tests): D and the codes of v[0..n). */
float lbo_xor_quantise(const float *v, int64_t n, int B, int64_t *codes)
{
    const float D = xor_scale(v, n, B);
    for (int64_t j = 0; j < n; ++j) codes[j] = xor_code(v[j], D);
    return D;
}
