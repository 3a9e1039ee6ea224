/*
 * kq_oracle.c -- plain, slow, scalar CPU oracle for the KroQuant online
 * activation quantizer and its two baselines.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test-suite, the package
 * smoke check and the benchmark's CPU-baseline leg may load or call this
 * library.  It shares no code, header, table or helper with the CUDA path.
 *
 * Sources (cited by tag below):
 *   [KQ-abs]   "KroQuant: Kronecker-Structured Block Transforms for Efficient
 *              Post-Training Quantization of Diffusion Transformers"
 *              (arXiv 2607.21446), abstract: a learned invertible transform is
 *              applied to every 32-element block of each activation row, the
 *              result is quantized to MXFP4 (W4A4, "MXFP4e2"); SmoothQuant
 *              per-channel scaling is the cheap baseline.
 *   [KQ-Eq4]   Pith review of arXiv 2607.21446, skeptic critique on paper
 *              section 3.2, Eq. (4), and "key machinery": T is block diagonal,
 *              each 32x32 block K^(j) = G1 (x) G2 (x) G3 (x) G4 (x) G5 with 2x2 G_k;
 *              the inverse is folded into the weights offline.
 *   [KQ-Eq6]   Pith review of arXiv 2607.21446, referee note on paper section
 *              3.2, Eq. (6): each factor is G_k = L_k U_k with
 *              U_k = [[a_k, b_k], [0, -1/a_k]], three scalars per factor, 15
 *              per block; the Hadamard transform is the initialisation.
 *   [KQ-FWHT]  KroQuant abstract and the Pith review's "forward implications":
 *              fixed Hadamard transforms (applied by a fast Walsh-Hadamard
 *              transform) are the comparison point of the on-the-fly kernel.
 *   [OCP-MX]   OCP Microscaling Formats (MX) Specification v1.0, section 6.3
 *              (the MXFP4 block-32 conversion): shared scale
 *              2^(floor(log2(amax)) - emax_elem) with emax_elem = 2 for E2M1,
 *              stored as E8M0 (biased by 127); elements FP4 E2M1 with values
 *              {0, 0.5, 1, 1.5, 2, 3, 4, 6}, round-to-nearest-even, saturating.
 *   [SF]       NVIDIA PTX ISA, tcgen05 block-scaled MMA, the scale-factor
 *              operand: scale bytes of 128 consecutive rows x 4 consecutive
 *              32-blocks form one 512-byte unit, seen as 32 lanes x 16 bytes;
 *              lane l holds the rows l, l+32, l+64, l+96 (4 bytes each, in
 *              that order), each as the 4 blocks in increasing order.
 *
 * Readings taken where the sources are silent (each one is listed in the
 * design notes of the repository):
 *   R1 Kronecker index order is the textbook one:
 *      (A (x) B)[i*m + p][l*m + q] = A[i][l] * B[p][q], so G1 acts on bit 4
 *      (the most significant bit) of the in-block index and G5 on bit 0.
 *   R2 y = T x is evaluated once in double and rounded once to fp32; the block
 *      amax is taken over those fp32 values.
 *   R3 amax == 0 gives the clamped exponent -127 (scale byte 0x00); a block
 *      with a non-finite value gets scale byte 0xFF (out of contract).
 *   R4 The sign of an e2m1 code follows the sign bit of the scaled value, as
 *      IEEE rounding does, so a negative value that rounds to zero gives the
 *      code 0x8 ("-0").
 *   R5 Two codes per byte, the even element in the low nibble.
 *   R6 Factor storage: factors[j][k][r][c] (float32, 20 per block column j),
 *      k = 0..4 is G1..G5; "shared" mode uses one set for every column.
 *   R7 LU storage: params[j][k][3] = (a, b, c) of G_(k+1), L unit lower
 *      triangular.
 *   R9 The producer the quantizer is fused into is the DiT block's
 *      pre-linear normalisation: LayerNorm without affine over the d channels
 *      of a token row (mean, biased variance, eps inside the square root),
 *      then AdaLN modulation x_mod = LN(h) (1 + gamma_b) + beta_b with
 *      per-sample vectors gamma_b, beta_b of length d; rows are grouped by
 *      sample, M / nsamples consecutive rows per sample.  x_mod is not rounded
 *      to bf16 (nothing is written between the two steps).
 *   R10 The W4A4 linear layer (the step after the quantizer, [KQ-abs]: both
 *      operands in MXFP4) computes D[m][n] = sum_k a[m][k] b[n][k] with a and b
 *      the decoded MXFP4 values of X T^T and W T^-1 ([KQ-Eq4]); D is exact in
 *      double here.  Its scale bytes may be stored in the scale-factor layout
 *      of the block-scaled tensor-core MMA ([SF] below).
 *   R8 The fixed-Hadamard baseline of block size H (a power of two, 32 <= H,
 *      H | d) is the orthonormal Sylvester transform H_H / sqrt(H) on every
 *      H consecutive channels, followed by the same MX quantizer (blocks of
 *      32 inside each H-block).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define BLK 32

int oracle_abi_version(void) { return 1; }

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* A bf16 value is the upper 16 bits of an IEEE binary32. */
static double bf16_value(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* [KQ-Eq4] + R1: K[i][l] = prod_k G_k[bit_(4-k)(i)][bit_(4-k)(l)], in double. */
static void kron_expand_d(const double *F /* [5][2][2] */, double *K /* [32][32] */)
{
    for (int i = 0; i < BLK; ++i) {
        for (int l = 0; l < BLK; ++l) {
            double p = 1.0;
            for (int k = 0; k < 5; ++k) {
                int bi = (i >> (4 - k)) & 1;
                int bl = (l >> (4 - k)) & 1;
                p *= F[k * 4 + bi * 2 + bl];
            }
            K[i * BLK + l] = p;
        }
    }
}

void oracle_kron_expand(const float *F /* [5][2][2] */, double *K /* [32][32] */)
{
    double Fd[20];
    for (int e = 0; e < 20; ++e) Fd[e] = (double)F[e];
    kron_expand_d(Fd, K);
}

/* [KQ-Eq6] LU form of one factor: G = L U with U = [[a, b], [0, -1/a]] and
 * L = [[1, 0], [c, 1]] (reading: L is unit lower triangular), so
 * G = [[a, b], [c a, c b - 1/a]] and det G = -1.  In double. */
void oracle_lu_factor(double a, double b, double c, double *G /* [2][2] */)
{
    G[0] = a;
    G[1] = b;
    G[2] = c * a;
    G[3] = c * b - 1.0 / a;
}

/* K from the 15 LU scalars of one block: params[k] = (a_k, b_k, c_k) of G_(k+1). */
void oracle_kron_expand_lu(const float *params /* [5][3] */, double *K /* [32][32] */)
{
    double Fd[20];
    for (int k = 0; k < 5; ++k)
        oracle_lu_factor((double)params[3 * k], (double)params[3 * k + 1], (double)params[3 * k + 2], Fd + 4 * k);
    kron_expand_d(Fd, K);
}

/* Dense inverse of a 32x32 matrix by Gauss-Jordan elimination with partial
 * pivoting, in double.  Returns 0 on success, -1 if a pivot is exactly 0. */
int oracle_inverse32(const double *A, double *Ainv)
{
    double a[BLK][2 * BLK];
    for (int i = 0; i < BLK; ++i) {
        for (int j = 0; j < BLK; ++j) {
            a[i][j] = A[i * BLK + j];
            a[i][BLK + j] = (i == j) ? 1.0 : 0.0;
        }
    }
    for (int c = 0; c < BLK; ++c) {
        int piv = c;
        for (int r = c + 1; r < BLK; ++r)
            if (fabs(a[r][c]) > fabs(a[piv][c])) piv = r;
        if (a[piv][c] == 0.0) return -1;
        if (piv != c) {
            for (int j = 0; j < 2 * BLK; ++j) {
                double t = a[c][j];
                a[c][j] = a[piv][j];
                a[piv][j] = t;
            }
        }
        double inv = 1.0 / a[c][c];
        for (int j = 0; j < 2 * BLK; ++j) a[c][j] *= inv;
        for (int r = 0; r < BLK; ++r) {
            if (r == c) continue;
            double f = a[r][c];
            if (f == 0.0) continue;
            for (int j = 0; j < 2 * BLK; ++j) a[r][j] -= f * a[c][j];
        }
    }
    for (int i = 0; i < BLK; ++i)
        for (int j = 0; j < BLK; ++j) Ainv[i * BLK + j] = a[i][BLK + j];
    return 0;
}

/* [OCP-MX] E8M0 shared-scale byte from the block amax (fp32), with R3.
 * floor(log2(amax)) is read off frexp exactly (no log2 call):
 * amax = m * 2^ex with 0.5 <= m < 1, so floor(log2(amax)) = ex - 1. */
uint8_t oracle_e8m0(float amax)
{
    if (!isfinite(amax)) return 0xFF;
    if (amax == 0.0f) return 0x00;
    int ex = 0;
    (void)frexp((double)amax, &ex);
    int e = (ex - 1) - 2;
    if (e < -127) e = -127;
    if (e > 127) e = 127;
    return (uint8_t)(e + 127);
}

/* [OCP-MX] FP4 E2M1 code of a scaled value: nearest grid magnitude by brute
 * force; on an exact tie the even code (magnitude LSB 0) wins; magnitudes
 * beyond 6 land on 6 (saturation); sign from the sign bit (R4). */
static const double E2M1_GRID[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

uint8_t oracle_e2m1(double v)
{
    double a = fabs(v);
    int best = 0;
    double bestd = fabs(a - E2M1_GRID[0]);
    for (int k = 1; k < 8; ++k) {
        double dk = fabs(a - E2M1_GRID[k]);
        if (dk < bestd || (dk == bestd && (k & 1) == 0)) {
            best = k;
            bestd = dk;
        }
    }
    uint8_t code = (uint8_t)best;
    if (signbit(v)) code |= 0x8;
    return code;
}

/* [OCP-MX] one 32-element block: amax over |y|, E8M0 byte, scaled values
 * v = y * 2^-e (exact in double), E2M1 codes packed two per byte (R5). */
void oracle_mx_block(const float *y /* [32] */, uint8_t *codes /* [16] */, uint8_t *scale)
{
    float amax = 0.0f;
    int finite = 1;
    for (int i = 0; i < BLK; ++i) {
        if (!isfinite(y[i])) finite = 0;
        float a = fabsf(y[i]);
        if (a > amax) amax = a;
    }
    uint8_t sb = finite ? oracle_e8m0(amax) : 0xFF;
    *scale = sb;
    if (sb == 0xFF) {
        memset(codes, 0, BLK / 2);
        return;
    }
    int e = (int)sb - 127;
    uint8_t c[BLK];
    for (int i = 0; i < BLK; ++i) c[i] = oracle_e2m1(ldexp((double)y[i], -e));
    for (int b = 0; b < BLK / 2; ++b)
        codes[b] = (uint8_t)(c[2 * b] | (c[2 * b + 1] << 4));
}

/* Expand every column's K^(j) once (nb x 1024 doubles), from generic factors
 * (20 floats per column) or, with lu != 0, from LU scalars (15 per column). */
static double *expand_all_mode(const float *params, int shared, int64_t nb, int lu)
{
    int64_t ncol = shared ? 1 : nb;
    double *K = (double *)malloc((size_t)ncol * BLK * BLK * sizeof(double));
    if (!K) return NULL;
    for (int64_t j = 0; j < ncol; ++j) {
        if (lu)
            oracle_kron_expand_lu(params + j * 15, K + j * BLK * BLK);
        else
            oracle_kron_expand(params + j * 20, K + j * BLK * BLK);
    }
    return K;
}

static double *expand_all(const float *factors, int shared, int64_t nb)
{
    return expand_all_mode(factors, shared, nb, 0);
}

/* [KQ-abs], [KQ-Eq4]: y = T x per 32-block of every row, dense matvec with the
 * expanded K^(j) summed in double and rounded once to fp32 (R2).  If absb is
 * not NULL it receives (|K^(j)| |x|)_i, the scale of the dot product's
 * rounding error, used by tests to form tolerances. */
int oracle_kq_transform(const uint16_t *x, const float *factors, int shared,
                        int64_t M, int64_t d, float *y, double *absb)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
    double *K = expand_all(factors, shared, nb);
    if (!K) return -5;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t j = 0; j < nb; ++j) {
            const double *Kj = K + (shared ? 0 : j) * BLK * BLK;
            const uint16_t *xb = x + r * d + j * BLK;
            double xv[BLK];
            for (int l = 0; l < BLK; ++l) xv[l] = bf16_value(xb[l]);
            for (int i = 0; i < BLK; ++i) {
                double s = 0.0, sa = 0.0;
                for (int l = 0; l < BLK; ++l) {
                    s += Kj[i * BLK + l] * xv[l];
                    sa += fabs(Kj[i * BLK + l]) * fabs(xv[l]);
                }
                y[r * d + j * BLK + i] = (float)s;
                if (absb) absb[r * d + j * BLK + i] = sa;
            }
        }
    }
    free(K);
    return 0;
}

/* The KroQuant quantizer: transform (above), then the MX block quantizer. */
int oracle_kq_quantize(const uint16_t *x, const float *factors, int shared,
                       int64_t M, int64_t d, uint8_t *codes, uint8_t *scales)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
    double *K = expand_all(factors, shared, nb);
    if (!K) return -5;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t j = 0; j < nb; ++j) {
            const double *Kj = K + (shared ? 0 : j) * BLK * BLK;
            const uint16_t *xb = x + r * d + j * BLK;
            double xv[BLK];
            float yv[BLK];
            for (int l = 0; l < BLK; ++l) xv[l] = bf16_value(xb[l]);
            for (int i = 0; i < BLK; ++i) {
                double s = 0.0;
                for (int l = 0; l < BLK; ++l) s += Kj[i * BLK + l] * xv[l];
                yv[i] = (float)s;
            }
            oracle_mx_block(yv, codes + r * (d / 2) + j * (BLK / 2), scales + r * nb + j);
        }
    }
    free(K);
    return 0;
}

/* [KQ-abs] SmoothQuant baseline: y_c = fp32(x_c * m_c) with the per-channel
 * multiplier m_c = 1/s_c given as input, then the MX block quantizer.  The
 * product of a bf16 and an fp32 value is exact in double, so the single
 * rounding to fp32 is the correctly rounded fp32 product. */
int oracle_sq_quantize(const uint16_t *x, const float *mult, int64_t M, int64_t d,
                       uint8_t *codes, uint8_t *scales)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t j = 0; j < nb; ++j) {
            float yv[BLK];
            for (int i = 0; i < BLK; ++i) {
                int64_t c = j * BLK + i;
                yv[i] = (float)(bf16_value(x[r * d + c]) * (double)mult[c]);
            }
            oracle_mx_block(yv, codes + r * (d / 2) + j * (BLK / 2), scales + r * nb + j);
        }
    }
    return 0;
}

/* Plain MXFP4 baseline: no transform, the MX block quantizer on x itself. */
int oracle_mx_quantize(const uint16_t *x, int64_t M, int64_t d, uint8_t *codes, uint8_t *scales)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t j = 0; j < nb; ++j) {
            float yv[BLK];
            for (int i = 0; i < BLK; ++i) yv[i] = (float)bf16_value(x[r * d + j * BLK + i]);
            oracle_mx_block(yv, codes + r * (d / 2) + j * (BLK / 2), scales + r * nb + j);
        }
    }
    return 0;
}

/* [KQ-Eq4] offline fold of the inverse into the weights: W' = W T^-1, i.e.
 * for every row n and column block j, W'[n, blk j] = W[n, blk j] K^(j)^-1,
 * with K^(j)^-1 the Gauss-Jordan inverse of the dense expansion.  Summed in
 * double, rounded once to fp32.  If absb is not NULL it receives
 * (|W[n, blk j]| |K^(j)^-1|)_c for tolerances.  Returns -3 if some K^(j) is
 * singular. */
int oracle_fold_weights(const float *W, const float *factors, int shared,
                        float *Wout, double *absb, int64_t N, int64_t d)
{
    if (d % BLK != 0 || N < 0) return -2;
    int64_t nb = d / BLK;
    int64_t ncol = shared ? 1 : nb;
    double *K = expand_all(factors, shared, nb);
    if (!K) return -5;
    double *Ki = (double *)malloc((size_t)ncol * BLK * BLK * sizeof(double));
    if (!Ki) {
        free(K);
        return -5;
    }
    int bad = 0;
    for (int64_t j = 0; j < ncol; ++j)
        if (oracle_inverse32(K + j * BLK * BLK, Ki + j * BLK * BLK) != 0) bad = 1;
    free(K);
    if (bad) {
        free(Ki);
        return -3;
    }
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t j = 0; j < nb; ++j) {
            const double *Kij = Ki + (shared ? 0 : j) * BLK * BLK;
            const float *w = W + n * d + j * BLK;
            for (int c = 0; c < BLK; ++c) {
                double s = 0.0, sa = 0.0;
                for (int r = 0; r < BLK; ++r) {
                    s += (double)w[r] * Kij[r * BLK + c];
                    sa += fabs((double)w[r]) * fabs(Kij[r * BLK + c]);
                }
                Wout[n * d + j * BLK + c] = (float)s;
                if (absb) absb[n * d + j * BLK + c] = sa;
            }
        }
    }
    free(Ki);
    return 0;
}

/* The dense per-block transform with already expanded K (double), shared by
 * the generic-factor and LU entry points below. */
static void transform_with(const double *K, int shared, const uint16_t *x, int64_t M, int64_t d, float *y,
                           double *absb, uint8_t *codes, uint8_t *scales)
{
    int64_t nb = d / BLK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        for (int64_t j = 0; j < nb; ++j) {
            const double *Kj = K + (shared ? 0 : j) * BLK * BLK;
            double xv[BLK];
            float yv[BLK];
            for (int l = 0; l < BLK; ++l) xv[l] = bf16_value(x[r * d + j * BLK + l]);
            for (int i = 0; i < BLK; ++i) {
                double sacc = 0.0, sa = 0.0;
                for (int l = 0; l < BLK; ++l) {
                    sacc += Kj[i * BLK + l] * xv[l];
                    sa += fabs(Kj[i * BLK + l]) * fabs(xv[l]);
                }
                yv[i] = (float)sacc;
                if (y) y[r * d + j * BLK + i] = yv[i];
                if (absb) absb[r * d + j * BLK + i] = sa;
            }
            if (codes) oracle_mx_block(yv, codes + r * (d / 2) + j * (BLK / 2), scales + r * nb + j);
        }
    }
}

/* [KQ-Eq6] the KroQuant transform and quantizer from the 15 LU scalars per block. */
int oracle_kq_transform_lu(const uint16_t *x, const float *params, int shared, int64_t M, int64_t d, float *y,
                           double *absb)
{
    if (d % BLK != 0 || M < 0) return -2;
    double *K = expand_all_mode(params, shared, d / BLK, 1);
    if (!K) return -5;
    transform_with(K, shared, x, M, d, y, absb, NULL, NULL);
    free(K);
    return 0;
}

int oracle_kq_quantize_lu(const uint16_t *x, const float *params, int shared, int64_t M, int64_t d,
                          uint8_t *codes, uint8_t *scales)
{
    if (d % BLK != 0 || M < 0) return -2;
    double *K = expand_all_mode(params, shared, d / BLK, 1);
    if (!K) return -5;
    transform_with(K, shared, x, M, d, NULL, NULL, codes, scales);
    free(K);
    return 0;
}

static int popcount_u(unsigned v)
{
    int c = 0;
    while (v) {
        c += (int)(v & 1u);
        v >>= 1;
    }
    return c;
}

/* [KQ-FWHT] + R8: y = H_H x / sqrt(H) on every H-block, H[i][f] = (-1)^popcount(i & f)
 * (the Sylvester matrix), summed in double and rounded once to fp32; then the
 * MX quantizer on each 32-block.  absb receives (|H_H| |x|)_i / sqrt(H). */
int oracle_fwht_transform(const uint16_t *x, int64_t H, int64_t M, int64_t d, float *y, double *absb,
                          uint8_t *codes, uint8_t *scales)
{
    if (H < BLK || (H & (H - 1)) != 0 || d % H != 0 || M < 0) return -2;
    const double inv = 1.0 / sqrt((double)H);
    int64_t nb = d / BLK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        double *xv = (double *)malloc((size_t)H * sizeof(double));
        float *yv = (float *)malloc((size_t)H * sizeof(float));
        for (int64_t h0 = 0; h0 < d; h0 += H) {
            for (int64_t f = 0; f < H; ++f) xv[f] = bf16_value(x[r * d + h0 + f]);
            for (int64_t i = 0; i < H; ++i) {
                double sacc = 0.0, sa = 0.0;
                for (int64_t f = 0; f < H; ++f) {
                    double hv = (popcount_u((unsigned)(i & f)) & 1) ? -1.0 : 1.0;
                    sacc += hv * xv[f];
                    sa += fabs(xv[f]);
                }
                yv[i] = (float)(sacc * inv);
                if (y) y[r * d + h0 + i] = yv[i];
                if (absb) absb[r * d + h0 + i] = sa * inv;
            }
            if (codes)
                for (int64_t b = 0; b < H / BLK; ++b)
                    oracle_mx_block(yv + b * BLK, codes + r * (d / 2) + (h0 / 2) + b * (BLK / 2),
                                    scales + r * nb + h0 / BLK + b);
        }
        free(xv);
        free(yv);
    }
    return 0;
}

/* [OCP-MX] MXFP4 decode: value = E2M1(code) * 2^(byte - 127); byte 0xFF is NaN. */
int oracle_mx_dequantize(const uint8_t *codes, const uint8_t *scales, int64_t M, int64_t d, float *out)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
    for (int64_t r = 0; r < M; ++r)
        for (int64_t j = 0; j < nb; ++j) {
            uint8_t sb = scales[r * nb + j];
            for (int i = 0; i < BLK; ++i) {
                uint8_t byte = codes[r * (d / 2) + j * (BLK / 2) + i / 2];
                uint8_t c = (i & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
                double v = E2M1_GRID[c & 7];
                if (c & 8) v = -v;
                out[r * d + j * BLK + i] = (sb == 0xFF) ? (float)NAN : (float)ldexp(v, (int)sb - 127);
            }
        }
    return 0;
}

/* x = K^(j)^-1 y on every 32-block (Gauss-Jordan inverse of the dense K, in
 * double, rounded once); absb receives (|K^-1| |y|)_i. */
int oracle_kq_inverse(const float *y, const float *factors, int shared, int64_t M, int64_t d, float *x, double *absb)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
    int64_t ncol = shared ? 1 : nb;
    double *K = expand_all(factors, shared, nb);
    if (!K) return -5;
    double *Ki = (double *)malloc((size_t)ncol * BLK * BLK * sizeof(double));
    if (!Ki) {
        free(K);
        return -5;
    }
    int bad = 0;
    for (int64_t j = 0; j < ncol; ++j)
        if (oracle_inverse32(K + j * BLK * BLK, Ki + j * BLK * BLK) != 0) bad = 1;
    free(K);
    if (bad) {
        free(Ki);
        return -3;
    }
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r)
        for (int64_t j = 0; j < nb; ++j) {
            const double *Kij = Ki + (shared ? 0 : j) * BLK * BLK;
            for (int i = 0; i < BLK; ++i) {
                double sacc = 0.0, sa = 0.0;
                for (int l = 0; l < BLK; ++l) {
                    double yv = (double)y[r * d + j * BLK + l];
                    sacc += Kij[i * BLK + l] * yv;
                    sa += fabs(Kij[i * BLK + l]) * fabs(yv);
                }
                x[r * d + j * BLK + i] = (float)sacc;
                if (absb) absb[r * d + j * BLK + i] = sa;
            }
        }
    free(Ki);
    return 0;
}

/* [KQ-abs] "normalization layers ... force this transform to run online": the
 * quantizer fused with the normalisation that produces its input (R9).  In
 * double: mu, var over the row, x_mod, then y = K x_mod per block, rounded once
 * to fp32; absb = (|K| |x_mod|)_i; codes/scales by the MX quantizer. */
int oracle_norm_kq(const uint16_t *h, const float *gamma, const float *beta, int64_t nsamples, double eps,
                   const float *factors, int shared, int64_t M, int64_t d, float *y, double *absb,
                   uint8_t *codes, uint8_t *scales)
{
    if (d % BLK != 0 || M < 0 || nsamples <= 0 || M % nsamples != 0) return -2;
    int64_t nb = d / BLK;
    int64_t rows_per = M / nsamples;
    double *K = expand_all(factors, shared, nb);
    if (!K) return -5;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r) {
        const int64_t b = r / rows_per;
        double *xm = (double *)malloc((size_t)d * sizeof(double));
        double mu = 0.0, var = 0.0;
        for (int64_t c = 0; c < d; ++c) mu += bf16_value(h[r * d + c]);
        mu /= (double)d;
        for (int64_t c = 0; c < d; ++c) {
            double t = bf16_value(h[r * d + c]) - mu;
            var += t * t;
        }
        var /= (double)d;
        double inv = 1.0 / sqrt(var + eps);
        for (int64_t c = 0; c < d; ++c)
            xm[c] = (bf16_value(h[r * d + c]) - mu) * inv * (1.0 + (double)gamma[b * d + c]) + (double)beta[b * d + c];
        for (int64_t j = 0; j < nb; ++j) {
            const double *Kj = K + (shared ? 0 : j) * BLK * BLK;
            float yv[BLK];
            for (int i = 0; i < BLK; ++i) {
                double sacc = 0.0, sa = 0.0;
                for (int l = 0; l < BLK; ++l) {
                    sacc += Kj[i * BLK + l] * xm[j * BLK + l];
                    sa += fabs(Kj[i * BLK + l]) * fabs(xm[j * BLK + l]);
                }
                yv[i] = (float)sacc;
                if (y) y[r * d + j * BLK + i] = yv[i];
                if (absb) absb[r * d + j * BLK + i] = sa;
            }
            if (codes) oracle_mx_block(yv, codes + r * (d / 2) + j * (BLK / 2), scales + r * nb + j);
        }
        free(xm);
    }
    free(K);
    return 0;
}

/* [SF] byte offset of the scale of row r, block column j, for a matrix with
 * nb block columns: 512-byte units ordered row-unit major, the ceil(nb/4)
 * units of one 128-row group consecutive; inside a unit as stated above. */
int64_t oracle_sf_offset(int64_t r, int64_t j, int64_t nb)
{
    int64_t ka = (nb + 3) / 4;
    int64_t unit = (r / 128) * ka + j / 4;
    int64_t lane = r % 32, group = (r % 128) / 32;
    return unit * 512 + lane * 16 + group * 4 + (j % 4);
}

int64_t oracle_sf_bytes(int64_t rows, int64_t nb)
{
    return ((rows + 127) / 128) * ((nb + 3) / 4) * 512;
}

/* Row-major scales [rows][nb] -> [SF] layout.  With nb odd the byte of block
 * column nb (padding inside the last unit) is set to 0x00 (2^-127, finite):
 * a K=64 step of the MMA reads two consecutive block columns, and the last
 * one then pairs the real column nb-1 with this pad.  Other padding bytes
 * are left as they are. */
int oracle_scales_to_sf(const uint8_t *scales, int64_t rows, int64_t nb, uint8_t *sf)
{
    if (rows < 0 || nb <= 0) return -2;
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t j = 0; j < nb; ++j) sf[oracle_sf_offset(r, j, nb)] = scales[r * nb + j];
        if (nb & 1) sf[oracle_sf_offset(r, nb, nb)] = 0x00;
    }
    return 0;
}

/* [OCP-MX] the plain MXFP4 quantizer on fp32 input (the folded weights
 * W T^-1 of [KQ-Eq4] are fp32). */
int oracle_mx_quantize_f32(const float *x, int64_t M, int64_t d, uint8_t *codes, uint8_t *scales)
{
    if (d % BLK != 0 || M < 0) return -2;
    int64_t nb = d / BLK;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < M; ++r)
        for (int64_t j = 0; j < nb; ++j)
            oracle_mx_block(x + r * d + j * BLK, codes + r * (d / 2) + j * (BLK / 2), scales + r * nb + j);
    return 0;
}

/* One decoded MXFP4 element (R5 nibble order, [OCP-MX] value), in double. */
static double mx_value(const uint8_t *codes, const uint8_t *scales, int64_t r, int64_t k, int64_t K)
{
    uint8_t byte = codes[r * (K / 2) + k / 2];
    uint8_t c = (k & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0xF);
    double v = E2M1_GRID[c & 7];
    if (c & 8) v = -v;
    uint8_t sb = scales[r * (K / BLK) + k / BLK];
    return sb == 0xFF ? NAN : ldexp(v, (int)sb - 127);
}

/* R10: D[m][n] = sum_k a[m][k] b[n][k] over the decoded operands (row-major
 * scales), summed in double.  Each product is exact (E2M1 values carry at
 * most 2 significant bits, scales are powers of two); the double sum rounds
 * far below any fp32 accumulation.  If absd is not NULL it receives
 * sum_k |a[m][k] b[n][k]| for tolerances.  Rows ms[0..nm) of A only when ms
 * is not NULL (sampled checks); D and absd are then [nm][N]. */
int oracle_mxf4_gemm(const uint8_t *ca, const uint8_t *sa, const uint8_t *cb, const uint8_t *sbb,
                     const int64_t *ms, int64_t nm, int64_t M, int64_t N, int64_t K, double *D, double *absd)
{
    if (K <= 0 || K % BLK != 0 || M < 0 || N < 0) return -2;
    int64_t rows = ms ? nm : M;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < rows; ++i) {
        int64_t m = ms ? ms[i] : i;
        if (m < 0 || m >= M) continue;
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = mx_value(ca, sa, m, k, K) * mx_value(cb, sbb, n, k, K);
                acc += p;
                aacc += fabs(p);
            }
            D[i * N + n] = acc;
            if (absd) absd[i * N + n] = aacc;
        }
    }
    return 0;
}
