/*
 * oracle.c -- plain, slow, fp64 CPU definition of the AXELRAM write and read path.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg call this file.  The CUDA library never links it, and this file
 * includes nothing from the library: the two share no code, tables or constants.
 *
 * Source: "AXELRAM: Quantize Once, Never Dequantize" (arXiv 2604.02638), abstract,
 * as printed on its fugumt.com summary pages; the codebook solver names listed for
 * that paper's repository on its codewithpapers.app record (axelram/quantize/codebook.py:
 * _target_pdf, _conditional_mean, solve_lloyd_max).  The abstract fixes *what* is
 * computed only in words:
 *   - an orthogonal transform concentrates every coordinate of a rotated unit key
 *     to N(0, 1/d);
 *   - hence the optimal scalar quantizer is a design-time codebook that depends
 *     only on the head dimension d and the bit width b;
 *   - keys are transformed on write; scores are read by table lookup with no
 *     inverse transform;
 *   - the transform carries a (seeded) sign pattern.
 * The plainest concrete reading, used here and stated step by step:
 *   R = H * diag(D) / sqrt(d), H the Sylvester-ordered Walsh-Hadamard matrix,
 *   D in {+1,-1}^d; u = R k / ||k|| with ||k|| the stored (fp32) norm;
 *   codebook = Lloyd-Max quantizer of N(0,1) scaled by 1/sqrt(d), rounded to fp32;
 *   idx_j = nearest centroid to u_j (ties to the lower index);
 *   idx packed as a dense LSB-first bit stream, d*b/8 bytes per key;
 *   q' = R q;  score = ||k|| * sum_j q'_j * c[idx_j] / sqrt(d).
 *
 * Everything is fp64 except what the method stores: centroids, boundaries and
 * norms are rounded to fp32 because that is what a cache holds.
 *
 * Parity pins for every function live in tests/test_oracle_pins.py.  The one
 * figure of the pages that no function here reproduces -- the abstract's 102.4-fold
 * cut in multiplications per query -- is parity unpinned: the pages give no
 * derivation of it.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_PI 3.14159265358979323846

#define ORACLE_OK 0
#define ORACLE_EINVAL (-1)

static int is_pow2(int d) { return d >= 1 && (d & (d - 1)) == 0; }

static int bit_count(unsigned x)
{
    int c = 0;
    while (x) {
        c += (int)(x & 1u);
        x >>= 1;
    }
    return c;
}

/*
 * Sylvester-ordered Walsh-Hadamard matrix, d x d, row-major:
 *   H[i][j] = (-1)^popcount(i AND j).
 * This is the closed form of Sylvester's doubling H_2n = [[H_n, H_n], [H_n, -H_n]]
 * (AXELRAM abstract: the quantizer works on orthogonally transformed keys; the
 * Walsh-Hadamard choice and its natural order are this oracle's reading).
 */
int oracle_hadamard(int d, double *H)
{
    if (!is_pow2(d) || !H) return ORACLE_EINVAL;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
            H[(size_t)i * d + j] = (bit_count((unsigned)(i & j)) & 1) ? -1.0 : 1.0;
    return ORACLE_OK;
}

/*
 * The write-side transform R = H * diag(D) / sqrt(d), d x d, row-major.
 * signs[j] is D_j, +1 or -1 (AXELRAM abstract: the transform's sign pattern).
 * R is orthonormal, so it keeps norms and needs no inverse on the read side.
 */
int oracle_rotation(int d, const int8_t *signs, double *R)
{
    if (!is_pow2(d) || !signs || !R) return ORACLE_EINVAL;
    for (int j = 0; j < d; ++j)
        if (signs[j] != 1 && signs[j] != -1) return ORACLE_EINVAL;
    if (oracle_hadamard(d, R) != ORACLE_OK) return ORACLE_EINVAL;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j)
            R[(size_t)i * d + j] *= (double)signs[j] * inv_sqrt_d;
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Design-time codebook: Lloyd-Max quantizer of the standard normal.
 * --------------------------------------------------------------------------- */

/* standard normal density: the target pdf of every rotated unit-key coordinate
 * after scaling by sqrt(d) (AXELRAM abstract: coordinates concentrate to N(0,1/d)) */
static double std_normal_pdf(double x)
{
    if (isinf(x)) return 0.0;
    return exp(-0.5 * x * x) / sqrt(2.0 * ORACLE_PI);
}

/* P(a < X <= b) for X ~ N(0,1), written with erfc on the side that avoids
 * cancellation */
static double std_normal_mass(double a, double b)
{
    const double r2 = sqrt(2.0);
    if (b <= 0.0) return 0.5 * (erfc(-b / r2) - erfc(-a / r2));
    if (a >= 0.0) return 0.5 * (erfc(a / r2) - erfc(b / r2));
    return 1.0 - 0.5 * erfc(b / r2) - 0.5 * erfc(-a / r2);
}

/* E[X | a < X <= b] for X ~ N(0,1): (pdf(a) - pdf(b)) / P(a < X <= b) */
static double std_normal_conditional_mean(double a, double b)
{
    return (std_normal_pdf(a) - std_normal_pdf(b)) / std_normal_mass(a, b);
}

/*
 * Lloyd-Max quantizer of N(0,1) with L = 2^b levels, ascending, in fp64.
 * The two Lloyd-Max conditions are applied alternately until they hold:
 *   midpoint:  t_i = (c_i + c_{i+1}) / 2,                   i = 0 .. L-2
 *   centroid:  c_i = E[X | t_{i-1} < X <= t_i],  t_{-1} = -inf, t_{L-1} = +inf
 * Start: L evenly spaced points on (-3, 3).  The normal density is log-concave,
 * so the fixed point is unique and the start does not change the result.
 * Stop: when no centroid moves by more than 1e-15.
 * Returns the number of iterations through *iters (may be NULL).
 */
int oracle_lloyd_max_std(int b, double *c, int *iters)
{
    if (b < 1 || b > 8 || !c) return ORACLE_EINVAL;
    const int L = 1 << b;
    double t[256];
    double next[256];
    for (int i = 0; i < L; ++i) c[i] = -3.0 + 6.0 * (i + 0.5) / L;
    int it = 0;
    for (it = 1; it <= 1000000; ++it) {
        for (int i = 0; i + 1 < L; ++i) t[i] = 0.5 * (c[i] + c[i + 1]);
        double delta = 0.0;
        for (int i = 0; i < L; ++i) {
            const double lo = (i == 0) ? -INFINITY : t[i - 1];
            const double hi = (i == L - 1) ? INFINITY : t[i];
            next[i] = std_normal_conditional_mean(lo, hi);
            const double m = fabs(next[i] - c[i]);
            if (m > delta) delta = m;
        }
        memcpy(c, next, sizeof(double) * (size_t)L);
        if (delta <= 1e-15) break;
    }
    if (iters) *iters = it;
    return ORACLE_OK;
}

/*
 * The fp32 codebook for dimension d and bit width b, as a cache stores it:
 *   1. Lloyd-Max centroids of N(0,1) (above), made exactly symmetric:
 *      c_{L-1-i} = -c_i (the normal density is symmetric, so is its quantizer);
 *   2. scaled to N(0, 1/d) by sigma = 1/sqrt(d): a scale change of the density
 *      scales its Lloyd-Max quantizer by the same factor;
 *   3. rounded to fp32: centroids[L], ascending;
 *   4. decision boundaries[L-1] = fp32 of the exact midpoint of neighbouring
 *      fp32 centroids.
 * AXELRAM abstract: once rotated, the best quantizer is a function of d and b
 * alone, never of the data.
 */
int oracle_codebook(int d, int b, float *centroids, float *boundaries)
{
    if (!is_pow2(d) || b < 1 || b > 8 || !centroids) return ORACLE_EINVAL;
    const int L = 1 << b;
    double c[256];
    if (oracle_lloyd_max_std(b, c, NULL) != ORACLE_OK) return ORACLE_EINVAL;
    for (int i = 0; i < L / 2; ++i) {
        const double m = 0.5 * (c[L - 1 - i] - c[i]);
        c[i] = -m;
        c[L - 1 - i] = m;
    }
    const double sigma = 1.0 / sqrt((double)d);
    for (int i = 0; i < L; ++i) centroids[i] = (float)(c[i] * sigma);
    if (boundaries)
        for (int i = 0; i + 1 < L; ++i)
            boundaries[i] = (float)(0.5 * ((double)centroids[i] + (double)centroids[i + 1]));
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Packing of the b-bit indices of one key: a dense LSB-first bit stream.
 * Bit i of idx_j is bit (j*b + i) of the row; byte k of the row holds stream
 * bits 8k .. 8k+7, least significant first.  A row takes d*b/8 bytes.
 * (The pages say only that indices are stored; this layout is the reading.)
 * --------------------------------------------------------------------------- */

static void pack_row(const uint8_t *codes, int d, int b, uint8_t *row)
{
    const int P = d * b / 8;
    memset(row, 0, (size_t)P);
    for (int j = 0; j < d; ++j)
        for (int i = 0; i < b; ++i) {
            const int bit = j * b + i;
            if ((codes[j] >> i) & 1) row[bit / 8] |= (uint8_t)(1u << (bit % 8));
        }
}

static void unpack_row(const uint8_t *row, int d, int b, uint8_t *codes)
{
    for (int j = 0; j < d; ++j) {
        unsigned v = 0;
        for (int i = 0; i < b; ++i) {
            const int bit = j * b + i;
            v |= (unsigned)((row[bit / 8] >> (bit % 8)) & 1) << i;
        }
        codes[j] = (uint8_t)v;
    }
}

int oracle_pack(const uint8_t *codes, int64_t n, int d, int b, uint8_t *packed)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0) return ORACLE_EINVAL;
    const int P = d * b / 8;
    for (int64_t r = 0; r < n; ++r) pack_row(codes + r * d, d, b, packed + r * P);
    return ORACLE_OK;
}

int oracle_unpack(const uint8_t *packed, int64_t n, int d, int b, uint8_t *codes)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0) return ORACLE_EINVAL;
    const int P = d * b / 8;
    for (int64_t r = 0; r < n; ++r) unpack_row(packed + r * P, d, b, codes + r * d);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------
 * Write path: keys are transformed once, when they are stored.
 * --------------------------------------------------------------------------- */

/* norm and rotated unit vector of one key, R given (the steps of oracle_rotate_unit) */
static void rotate_unit_row(const double *R, const double *k, int d, float *norm_out, double *u)
{
    double ss = 0.0;
    for (int j = 0; j < d; ++j) ss += k[j] * k[j];
    const float norm = (float)sqrt(ss);
    *norm_out = norm;
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += R[(size_t)i * d + j] * k[j];
        u[i] = (norm > 0.0f) ? acc / (double)norm : 0.0;
    }
}

/*
 * Key norms and rotated unit keys.
 *   norms[r] = fp32( sqrt(sum_j K[r][j]^2) )      (stored per key)
 *   U[r]     = R K[r] / norms[r]                   (fp64; the stored norm is the
 *                                                   one the key is normalised by)
 * A zero key has norm 0 and U = 0 (reading: the pages do not cover it).
 * K: n x d fp64 (the caller upcasts bf16/fp16/fp32 inputs exactly).
 */
int oracle_rotate_unit(const double *K, int64_t n, int d, const int8_t *signs,
                       float *norms, double *U)
{
    if (!is_pow2(d) || n < 0 || !K || !signs || !norms || !U) return ORACLE_EINVAL;
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    if (!R) return ORACLE_EINVAL;
    if (oracle_rotation(d, signs, R) != ORACLE_OK) {
        free(R);
        return ORACLE_EINVAL;
    }
    for (int64_t r = 0; r < n; ++r) rotate_unit_row(R, K + r * d, d, norms + r, U + r * d);
    free(R);
    return ORACLE_OK;
}

/*
 * Scalar quantization of one rotated unit coordinate: the index of the nearest
 * fp32 centroid, by a linear scan in fp64, ties to the lower index.  *margin gets
 * the distance from u to the nearest decision point (exact midpoint of two
 * neighbouring centroids), the quantity the parity window is measured in.
 */
static int nearest_centroid(double u, const float *cent, int L, double *margin)
{
    int best = 0;
    double best_dist = fabs(u - (double)cent[0]);
    for (int l = 1; l < L; ++l) {
        const double dist = fabs(u - (double)cent[l]);
        if (dist < best_dist) {
            best = l;
            best_dist = dist;
        }
    }
    if (margin) {
        double m = INFINITY;
        for (int l = 0; l + 1 < L; ++l) {
            const double mid = 0.5 * ((double)cent[l] + (double)cent[l + 1]);
            const double dist = fabs(u - mid);
            if (dist < m) m = dist;
        }
        *margin = m;
    }
    return best;
}

/* quantize-on-write with the rotation R given (the steps of oracle_quantize) */
static int quantize_with(const double *K, int64_t n, int d, int b, const double *R, uint8_t *packed,
                         float *norms, double *margins)
{
    const int L = 1 << b;
    const int P = d * b / 8;
    float cent[256];
    if (oracle_codebook(d, b, cent, NULL) != ORACLE_OK) return ORACLE_EINVAL;
    double *u = (double *)malloc(sizeof(double) * (size_t)d);
    uint8_t *codes = (uint8_t *)malloc((size_t)d);
    if (!u || !codes) {
        free(u);
        free(codes);
        return ORACLE_EINVAL;
    }
    for (int64_t r = 0; r < n; ++r) {
        rotate_unit_row(R, K + r * d, d, norms + r, u);
        for (int j = 0; j < d; ++j)
            codes[j] = (uint8_t)nearest_centroid(u[j], cent, L, margins ? margins + r * d + j : NULL);
        pack_row(codes, d, b, packed + r * P);
    }
    free(u);
    free(codes);
    return ORACLE_OK;
}

/*
 * Quantize-on-write: keys K (n x d, fp64) -> packed indices (n x d*b/8 bytes)
 * and fp32 norms.  margins (n x d, may be NULL) receives, per coordinate, the
 * distance of u to its nearest decision point.
 * Steps, in the pages' order: sign flip and Walsh-Hadamard rotation, norm,
 * normalisation, nearest-centroid search on the design-time codebook, packing.
 */
int oracle_quantize(const double *K, int64_t n, int d, int b, const int8_t *signs,
                    uint8_t *packed, float *norms, double *margins)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0 || !K || !signs || !packed || !norms)
        return ORACLE_EINVAL;
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    if (!R || oracle_rotation(d, signs, R) != ORACLE_OK) {
        free(R);
        return ORACLE_EINVAL;
    }
    const int rc = quantize_with(K, n, d, b, R, packed, norms, margins);
    free(R);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Read path: scores come from table lookups on the stored indices; the keys are
 * never transformed back.
 * --------------------------------------------------------------------------- */

/* scores with the rotation R given (the steps of oracle_scores) */
static int scores_with(const double *q, const uint8_t *packed, const float *norms, int64_t n, int heads,
                       int group, int d, int b, const double *R, double *scores)
{
    const int P = d * b / 8;
    float cent[256];
    if (oracle_codebook(d, b, cent, NULL) != ORACLE_OK) return ORACLE_EINVAL;
    double *qr = (double *)malloc(sizeof(double) * (size_t)d);
    uint8_t *codes = (uint8_t *)malloc((size_t)d);
    if (!qr || !codes) {
        free(qr);
        free(codes);
        return ORACLE_EINVAL;
    }
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int h = 0; h < heads; ++h)
        for (int g = 0; g < group; ++g) {
            const double *qv = q + ((int64_t)h * group + g) * d;
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += R[(size_t)i * d + j] * qv[j];
                qr[i] = acc;
            }
            double *out = scores + ((int64_t)h * group + g) * n;
            for (int64_t t = 0; t < n; ++t) {
                unpack_row(packed + ((int64_t)h * n + t) * P, d, b, codes);
                double s = 0.0;
                for (int j = 0; j < d; ++j) s += qr[j] * (double)cent[codes[j]];
                out[t] = (double)norms[(int64_t)h * n + t] * s * inv_sqrt_d;
            }
        }
    free(qr);
    free(codes);
    return ORACLE_OK;
}

/*
 * Scores of every query against every quantized key of its KV head.
 *   q:      (heads*group) x d, fp64; query head h*group + g reads KV head h
 *   packed: heads x n x (d*b/8) bytes;  norms: heads x n (fp32)
 *   scores: (heads*group) x n, fp64
 * For each query: q' = R q once (no inverse transform on the keys), then
 *   score[t] = norms[t] * sum_j q'_j * c[idx_t[j]] / sqrt(d).
 * The 1/sqrt(d) is the attention temperature, separate from the one inside R.
 */
int oracle_scores(const double *q, const uint8_t *packed, const float *norms, int64_t n,
                  int heads, int group, int d, int b, const int8_t *signs, double *scores)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0 || heads < 1 || group < 1 || !q ||
        !packed || !norms || !signs || !scores)
        return ORACLE_EINVAL;
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    if (!R || oracle_rotation(d, signs, R) != ORACLE_OK) {
        free(R);
        return ORACLE_EINVAL;
    }
    const int rc = scores_with(q, packed, norms, n, heads, group, d, b, R, scores);
    free(R);
    return rc;
}

/* dequantized scores with the rotation R given (the steps of oracle_dequant_scores) */
static int dequant_scores_with(const double *q, const uint8_t *packed, const float *norms, int64_t n,
                               int heads, int group, int d, int b, const double *R, double *scores)
{
    const int P = d * b / 8;
    float cent[256];
    if (oracle_codebook(d, b, cent, NULL) != ORACLE_OK) return ORACLE_EINVAL;
    double *khat = (double *)malloc(sizeof(double) * (size_t)d);
    uint8_t *codes = (uint8_t *)malloc((size_t)d);
    if (!khat || !codes) {
        free(khat);
        free(codes);
        return ORACLE_EINVAL;
    }
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int h = 0; h < heads; ++h)
        for (int64_t t = 0; t < n; ++t) {
            unpack_row(packed + ((int64_t)h * n + t) * P, d, b, codes);
            const double nk = (double)norms[(int64_t)h * n + t];
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) acc += R[(size_t)i * d + j] * (double)cent[codes[i]];
                khat[j] = nk * acc;
            }
            for (int g = 0; g < group; ++g) {
                const double *qv = q + ((int64_t)h * group + g) * d;
                double s = 0.0;
                for (int j = 0; j < d; ++j) s += qv[j] * khat[j];
                scores[((int64_t)h * group + g) * n + t] = s * inv_sqrt_d;
            }
        }
    free(khat);
    free(codes);
    return ORACLE_OK;
}

/*
 * The same scores the long way, for the cross-check that table lookup without an
 * inverse transform equals attention on dequantized keys:
 *   k_hat_t = norms[t] * R^T c[idx_t],   score[t] = q . k_hat_t / sqrt(d).
 */
int oracle_dequant_scores(const double *q, const uint8_t *packed, const float *norms,
                          int64_t n, int heads, int group, int d, int b,
                          const int8_t *signs, double *scores)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0 || heads < 1 || group < 1 || !q ||
        !packed || !norms || !signs || !scores)
        return ORACLE_EINVAL;
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    if (!R || oracle_rotation(d, signs, R) != ORACLE_OK) {
        free(R);
        return ORACLE_EINVAL;
    }
    const int rc = dequant_scores_with(q, packed, norms, n, heads, group, d, b, R, scores);
    free(R);
    return rc;
}

/* ---------------------------------------------------------------------------
 * Block rotation (IsoQuant, arXiv 2603.28430, abstract), an alternative write
 * transform: the d coordinates split into d/4 blocks of 4, each read as a
 * quaternion v = v0 + v1 i + v2 j + v3 k, and T(v) = qL v conj(qR) with one
 * pair of unit quaternions per block (IsoQuant-Full; qR = 1 is IsoQuant-Fast).
 * The write and read steps are those above with R = T.
 * --------------------------------------------------------------------------- */

/* Hamilton product out = a b, with i^2 = j^2 = k^2 = ijk = -1 */
static void quat_mul(const double *a, const double *b, double *out)
{
    out[0] = a[0] * b[0] - a[1] * b[1] - a[2] * b[2] - a[3] * b[3];
    out[1] = a[0] * b[1] + a[1] * b[0] + a[2] * b[3] - a[3] * b[2];
    out[2] = a[0] * b[2] - a[1] * b[3] + a[2] * b[0] + a[3] * b[1];
    out[3] = a[0] * b[3] + a[1] * b[2] - a[2] * b[1] + a[3] * b[0];
}

/*
 * T as a dense d x d matrix.  quats: (d/4) x 8 doubles, block m's qL then qR
 * (w, x, y, z each).  Column 4m + c is T applied to the basis quaternion e_c of
 * block m; every entry outside the diagonal blocks is 0.
 */
int oracle_block_rotation(int d, const double *quats, double *R)
{
    if (d < 4 || d % 4 || !quats || !R) return ORACLE_EINVAL;
    for (size_t i = 0; i < (size_t)d * d; ++i) R[i] = 0.0;
    for (int m = 0; m < d / 4; ++m) {
        const double *qL = quats + 8 * m, *qR = quats + 8 * m + 4;
        const double qRc[4] = {qR[0], -qR[1], -qR[2], -qR[3]};
        for (int c = 0; c < 4; ++c) {
            double e[4] = {0.0, 0.0, 0.0, 0.0}, w[4], y[4];
            e[c] = 1.0;
            quat_mul(qL, e, w);
            quat_mul(w, qRc, y);
            for (int r = 0; r < 4; ++r) R[(size_t)(4 * m + r) * d + 4 * m + c] = y[r];
        }
    }
    return ORACLE_OK;
}

static double *block_matrix(int d, const double *quats)
{
    double *R = (double *)malloc(sizeof(double) * (size_t)d * d);
    if (R && oracle_block_rotation(d, quats, R) != ORACLE_OK) {
        free(R);
        return NULL;
    }
    return R;
}

/* oracle_quantize with the block rotation in place of H diag(signs) / sqrt(d) */
int oracle_quantize_block(const double *K, int64_t n, int d, int b, const double *quats,
                          uint8_t *packed, float *norms, double *margins)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0 || !K || !quats || !packed || !norms)
        return ORACLE_EINVAL;
    double *R = block_matrix(d, quats);
    if (!R) return ORACLE_EINVAL;
    const int rc = quantize_with(K, n, d, b, R, packed, norms, margins);
    free(R);
    return rc;
}

/* oracle_scores with the queries rotated by the block rotation */
int oracle_scores_block(const double *q, const uint8_t *packed, const float *norms, int64_t n,
                        int heads, int group, int d, int b, const double *quats, double *scores)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0 || heads < 1 || group < 1 || !q ||
        !packed || !norms || !quats || !scores)
        return ORACLE_EINVAL;
    double *R = block_matrix(d, quats);
    if (!R) return ORACLE_EINVAL;
    const int rc = scores_with(q, packed, norms, n, heads, group, d, b, R, scores);
    free(R);
    return rc;
}

/* oracle_dequant_scores with the block rotation */
int oracle_dequant_scores_block(const double *q, const uint8_t *packed, const float *norms, int64_t n,
                                int heads, int group, int d, int b, const double *quats, double *scores)
{
    if (!is_pow2(d) || d < 8 || b < 1 || b > 8 || n < 0 || heads < 1 || group < 1 || !q ||
        !packed || !norms || !quats || !scores)
        return ORACLE_EINVAL;
    double *R = block_matrix(d, quats);
    if (!R) return ORACLE_EINVAL;
    const int rc = dequant_scores_with(q, packed, norms, n, heads, group, d, b, R, scores);
    free(R);
    return rc;
}
