/*
 * oracle.c -- TEST INFRASTRUCTURE ONLY. A plain, slow, float64 CPU statement
 * of what the HARP rotate + quantize path computes. Only the tests, the smoke
 * check and the benchmark's CPU-baseline leg load it; the CUDA library shares
 * no code, header, table or constant with it and never calls it.
 *
 * Sources (the pages' titles and sections):
 *  [HARP]  "HARP: Hadamard-Preconditioned Adaptive Rotation Processor for
 *          Extreme LLM Quantization" (gist.science, paper 2605.29843),
 *          section 2.1 "core architecture" (mixed-radix schedule, stride
 *          stages of block-diagonal orthogonal matrices), section 2.2
 *          (B = Q(theta) G, Sylvester / QR base mixer, Givens / Cayley,
 *          theta = 0 gives the fixed RHT), section 1 (RHT = random signs times
 *          a normalised Hadamard, exactly orthogonal), section 5 (exact change
 *          of basis: the full-precision model is preserved).
 *  [PQ]    "PolarQuant: Optimal Gaussian Weight Quantization via Hadamard
 *          Rotation for LLM Compression" (gist.science, paper 2603.29078),
 *          section 2 "methodology" (blocks, l2 normalisation, rotation, scale
 *          to N(0,1), Lloyd-Max centroids, int codes + fp16 norm + fp32
 *          centroid table, H^-1 = H), section 1 (absmax: linear map assuming a
 *          uniform distribution on [-alpha, alpha]).
 *
 * Readings where the pages are silent (each is listed with its reason in the
 * design notes):
 *  - index convention: s_t = prod_{u>t} b_u; stage t's group c = h*s_t + l
 *    holds coordinates h*b_t*s_t + k*s_t + l, k = 0..b_t-1, and
 *    y[h b s + k s + l] = sum_j B[t][c][k][j] x[h b s + j s + l].
 *    The processor is M = B_{m-1} ... B_0 D (signs first, stage 0 first);
 *    its inverse is D B_0^T ... B_{m-1}^T.
 *  - Lloyd-Max group scale s = sqrt(mean of squares) (PQ's l2 norm times
 *    sqrt(g) so the normalised coordinates are N(0,1)); absmax scale
 *    s = max|x| / (2^(b-1) - 1). Scales are stored as fp16 (round to nearest
 *    even, saturating at 65504) and codes are computed with the stored scale.
 *  - Lloyd-Max code = number of fp32 midpoints t_k with z > t_k (ties go to
 *    the lower code); absmax code = clamp(rint(z), -qmax, qmax) + 2^(b-1).
 *    A group whose stored scale is 0 gets the middle code (K/2 or 2^(b-1)).
 *  - packing: code i of a row at bits [b*i, b*i + b) of the row's
 *    little-endian bitstream; rows are cols*b/8 bytes apart.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_BAD 1

/* ------------------------------------------------------------------ processor */

/* stride of stage t: s_t = b_{t+1} * ... * b_{m-1}  [HARP 2.1] */
static int64_t orc_stride(int m, const int32_t *radix, int t)
{
    int64_t s = 1;
    for (int u = t + 1; u < m; ++u) s *= radix[u];
    return s;
}

/* Offset (in doubles) of stage t's blocks when all stages are concatenated;
 * stage t holds d/b_t groups of b_t x b_t row-major blocks (out k, in j). */
static int64_t orc_block_offset(int64_t d, const int32_t *radix, int t)
{
    int64_t off = 0;
    for (int u = 0; u < t; ++u) off += d * radix[u];
    return off;
}

/* One stride stage [HARP 2.1]: every group c gets its own b x b block.
 * transpose = 1 applies B^T (used by the inverse). */
static void orc_stage(int64_t d, int b, int64_t s, const double *blk, int transpose,
                      const double *x, double *y)
{
    int64_t H = d / ((int64_t)b * s);
    for (int64_t h = 0; h < H; ++h) {
        for (int64_t l = 0; l < s; ++l) {
            const double *B = blk + (h * s + l) * (int64_t)b * b;
            int64_t base = h * b * s + l;
            for (int k = 0; k < b; ++k) {
                double acc = 0.0;
                for (int j = 0; j < b; ++j) {
                    double bkj = transpose ? B[(int64_t)j * b + k] : B[(int64_t)k * b + j];
                    acc += bkj * x[base + j * s];
                }
                y[base + k * s] = acc;
            }
        }
    }
}

/* y = M x (inverse = 0) or y = M^T x (inverse = 1) for one vector of length d.
 * blocks: all stages concatenated; signs: [d] of +-1 or NULL (all +1). */
int orc_apply(int64_t d, int m, const int32_t *radix, const double *blocks,
              const double *signs, int inverse, const double *x, double *y)
{
    int64_t prod = 1;
    for (int t = 0; t < m; ++t) {
        if (radix[t] < 1) return ORC_BAD;
        prod *= radix[t];
    }
    if (prod != d) return ORC_BAD;
    double *a = (double *)malloc(sizeof(double) * d);
    double *b = (double *)malloc(sizeof(double) * d);
    if (!a || !b) { free(a); free(b); return ORC_BAD; }
    if (!inverse) {
        for (int64_t i = 0; i < d; ++i) a[i] = signs ? signs[i] * x[i] : x[i];
        for (int t = 0; t < m; ++t) {
            orc_stage(d, radix[t], orc_stride(m, radix, t),
                      blocks + orc_block_offset(d, radix, t), 0, a, b);
            double *tmp = a; a = b; b = tmp;
        }
        memcpy(y, a, sizeof(double) * d);
    } else {
        memcpy(a, x, sizeof(double) * d);
        for (int t = m - 1; t >= 0; --t) {
            orc_stage(d, radix[t], orc_stride(m, radix, t),
                      blocks + orc_block_offset(d, radix, t), 1, a, b);
            double *tmp = a; a = b; b = tmp;
        }
        for (int64_t i = 0; i < d; ++i) y[i] = signs ? signs[i] * a[i] : a[i];
    }
    free(a);
    free(b);
    return ORC_OK;
}

/* Right side: every row r of X [rows x cols] becomes M r  (X -> X M^T).
 * Rows are independent; with OpenMP they are spread over the host threads
 * (the arithmetic of each row is unchanged). */
int orc_rotate_rows(int64_t rows, int64_t cols, int m, const int32_t *radix,
                    const double *blocks, const double *signs, int inverse,
                    const double *X, double *Y)
{
    int st = ORC_OK;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t r = 0; r < rows; ++r) {
        if (orc_apply(cols, m, radix, blocks, signs, inverse, X + r * cols, Y + r * cols)) {
#pragma omp atomic write
            st = ORC_BAD;
        }
    }
    return st;
}

/* Left side: every column w of X [rows x cols] becomes M w  (X -> M X).
 * Columns are independent (OpenMP over columns, one gather buffer per
 * thread). */
int orc_rotate_cols(int64_t rows, int64_t cols, int m, const int32_t *radix,
                    const double *blocks, const double *signs, int inverse,
                    const double *X, double *Y)
{
    int st = ORC_OK;
#pragma omp parallel
    {
        double *u = (double *)malloc(sizeof(double) * rows);
        double *v = (double *)malloc(sizeof(double) * rows);
        if (!u || !v) {
#pragma omp atomic write
            st = ORC_BAD;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t c = 0; c < cols; ++c) {
            if (!u || !v) continue;
            for (int64_t r = 0; r < rows; ++r) u[r] = X[r * cols + c];
            if (orc_apply(rows, m, radix, blocks, signs, inverse, u, v)) {
#pragma omp atomic write
                st = ORC_BAD;
                continue;
            }
            for (int64_t r = 0; r < rows; ++r) Y[r * cols + c] = v[r];
        }
        free(u);
        free(v);
    }
    return st;
}

/* Host threads the oracle's row / column loops use (OpenMP); n <= 0 leaves
 * the setting unchanged. Returns the current maximum. */
int orc_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* Dense stage matrices for tiny d: S_t[i][i'] = B[t][c][k][j] where
 * i = h b s + k s + l and i' = h b s + j s + l; then M = S_{m-1} ... S_0 D,
 * multiplied out as explicit d x d matrices.  out: [d x d] row-major. */
int orc_dense(int64_t d, int m, const int32_t *radix, const double *blocks,
              const double *signs, double *out)
{
    if (d > 1024) return ORC_BAD;
    double *S = (double *)calloc((size_t)(d * d), sizeof(double));
    double *P = (double *)calloc((size_t)(d * d), sizeof(double));
    double *T = (double *)calloc((size_t)(d * d), sizeof(double));
    if (!S || !P || !T) { free(S); free(P); free(T); return ORC_BAD; }
    for (int64_t i = 0; i < d; ++i) P[i * d + i] = signs ? signs[i] : 1.0;  /* P = D */
    for (int t = 0; t < m; ++t) {
        int b = radix[t];
        int64_t s = orc_stride(m, radix, t);
        const double *blk = blocks + orc_block_offset(d, radix, t);
        memset(S, 0, sizeof(double) * d * d);
        for (int64_t h = 0; h < d / (b * s); ++h)
            for (int64_t l = 0; l < s; ++l)
                for (int k = 0; k < b; ++k)
                    for (int j = 0; j < b; ++j)
                        S[(h * b * s + k * s + l) * d + (h * b * s + j * s + l)] =
                            blk[((h * s + l) * b + k) * b + j];
        for (int64_t i = 0; i < d; ++i)           /* T = S P */
            for (int64_t q = 0; q < d; ++q) {
                double acc = 0.0;
                for (int64_t r = 0; r < d; ++r) acc += S[i * d + r] * P[r * d + q];
                T[i * d + q] = acc;
            }
        memcpy(P, T, sizeof(double) * d * d);
    }
    memcpy(out, P, sizeof(double) * d * d);
    free(S);
    free(P);
    free(T);
    return ORC_OK;
}

/* --------------------------------------------------------------- block makers */

/* Normalised Sylvester Hadamard of order b = 2^k [HARP 2.2, base mixer]:
 * H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]], then divide by sqrt(b). */
int orc_sylvester(int b, double *H)
{
    if (b < 1 || (b & (b - 1))) return ORC_BAD;
    H[0] = 1.0;
    for (int n = 1; n < b; n *= 2)
        for (int i = 0; i < n; ++i)
            for (int j = 0; j < n; ++j) {
                double v = H[i * b + j];
                H[i * b + (j + n)] = v;
                H[(i + n) * b + j] = v;
                H[(i + n) * b + (j + n)] = -v;
            }
    double sc = 1.0 / sqrt((double)b);
    for (int i = 0; i < b * b; ++i) H[i] *= sc;
    return ORC_OK;
}

/* Q factor of G = Q R with R's diagonal positive [HARP 2.1, QR fallback]:
 * Gram-Schmidt on the columns of G, each column orthogonalised twice against
 * the previous ones, then normalised. G, Q: b x b row-major. */
int orc_qr_q(int b, const double *G, double *Q)
{
    for (int c = 0; c < b; ++c) {
        for (int r = 0; r < b; ++r) Q[r * b + c] = G[r * b + c];
        for (int pass = 0; pass < 2; ++pass)
            for (int p = 0; p < c; ++p) {
                double dot = 0.0;
                for (int r = 0; r < b; ++r) dot += Q[r * b + p] * Q[r * b + c];
                for (int r = 0; r < b; ++r) Q[r * b + c] -= dot * Q[r * b + p];
            }
        double nrm = 0.0;
        for (int r = 0; r < b; ++r) nrm += Q[r * b + c] * Q[r * b + c];
        nrm = sqrt(nrm);
        if (nrm == 0.0) return ORC_BAD;
        for (int r = 0; r < b; ++r) Q[r * b + c] /= nrm;
    }
    return ORC_OK;
}

/* Cayley map [HARP 2.2, b > 2]: Q = (I - A)^-1 (I + A) for skew-symmetric A,
 * by Gaussian elimination with partial pivoting on [I - A | I + A]. */
int orc_cayley(int b, const double *A, double *Q)
{
    int n2 = 2 * b;
    double *M = (double *)malloc(sizeof(double) * b * n2);
    if (!M) return ORC_BAD;
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            double id = (i == j) ? 1.0 : 0.0;
            M[i * n2 + j] = id - A[i * b + j];
            M[i * n2 + b + j] = id + A[i * b + j];
        }
    for (int c = 0; c < b; ++c) {
        int piv = c;
        for (int r = c + 1; r < b; ++r)
            if (fabs(M[r * n2 + c]) > fabs(M[piv * n2 + c])) piv = r;
        if (M[piv * n2 + c] == 0.0) { free(M); return ORC_BAD; }
        if (piv != c)
            for (int j = 0; j < n2; ++j) {
                double t = M[c * n2 + j]; M[c * n2 + j] = M[piv * n2 + j]; M[piv * n2 + j] = t;
            }
        for (int r = c + 1; r < b; ++r) {
            double f = M[r * n2 + c] / M[c * n2 + c];
            for (int j = c; j < n2; ++j) M[r * n2 + j] -= f * M[c * n2 + j];
        }
    }
    for (int j = 0; j < b; ++j)            /* back substitution, column by column */
        for (int i = b - 1; i >= 0; --i) {
            double acc = M[i * n2 + b + j];
            for (int k = i + 1; k < b; ++k) acc -= M[i * n2 + k] * Q[k * b + j];
            Q[i * b + j] = acc / M[i * n2 + i];
        }
    free(M);
    return ORC_OK;
}

/* Givens rotation [HARP 2.2, b = 2]: [[cos a, -sin a], [sin a, cos a]]. */
void orc_givens(double a, double *Q)
{
    Q[0] = cos(a); Q[1] = -sin(a);
    Q[2] = sin(a); Q[3] = cos(a);
}

/* Base mixer G_b [HARP 2.1-2.2]: Sylvester for b = 2^k, else the Q factor of
 * the stage's fixed Gaussian. */
static int orc_base_mixer(int b, const double *base_gauss, double *G)
{
    if ((b & (b - 1)) == 0) return orc_sylvester(b, G);
    if (!base_gauss) return ORC_BAD;
    return orc_qr_q(b, base_gauss, G);
}

/* Blocks of one stage from the raw draws.
 *  kind 0 (hadamard): B_c = G_b for every group (theta = 0, HARP 2.2 init)
 *  kind 1 (qr):       B_c = Q of QR(gauss_c)
 *  kind 2 (cayley):   B_c = Q(theta_c) G_b with Q the Cayley map (b > 2) of
 *                     A = skew_scale * S_c, S_c skew-symmetric with the strict
 *                     upper triangle of gauss_c above the diagonal; for b = 2
 *                     the Givens rotation by angle skew_scale * gauss_c[0][1].
 * gauss: [n_groups][b][b]; out: [n_groups][b][b] row-major (out k, in j). */
int orc_stage_blocks(int kind, int b, int64_t n_groups, const double *gauss,
                     const double *base_gauss, double skew_scale, double *out)
{
    double *G = (double *)malloc(sizeof(double) * b * b);
    double *A = (double *)malloc(sizeof(double) * b * b);
    double *Qm = (double *)malloc(sizeof(double) * b * b);
    int st = ORC_OK;
    if (!G || !A || !Qm) { st = ORC_BAD; goto done; }
    if (kind != 1) {
        st = orc_base_mixer(b, base_gauss, G);
        if (st) goto done;
    }
    for (int64_t c = 0; c < n_groups; ++c) {
        double *B = out + c * (int64_t)b * b;
        const double *g = gauss ? gauss + c * (int64_t)b * b : NULL;
        if (kind == 0) {
            memcpy(B, G, sizeof(double) * b * b);
        } else if (kind == 1) {
            st = orc_qr_q(b, g, B);
            if (st) goto done;
        } else if (kind == 2) {
            if (b == 2) {
                orc_givens(skew_scale * g[1], Qm);
            } else {
                for (int i = 0; i < b; ++i)
                    for (int j = 0; j < b; ++j)
                        A[i * b + j] = (i < j) ? skew_scale * g[i * b + j]
                                     : (i > j) ? -skew_scale * g[j * b + i] : 0.0;
                st = orc_cayley(b, A, Qm);
                if (st) goto done;
            }
            for (int i = 0; i < b; ++i)            /* B = Q G */
                for (int j = 0; j < b; ++j) {
                    double acc = 0.0;
                    for (int k = 0; k < b; ++k) acc += Qm[i * b + k] * G[k * b + j];
                    B[i * b + j] = acc;
                }
        } else {
            st = ORC_BAD;
            goto done;
        }
    }
done:
    free(G);
    free(A);
    free(Qm);
    return st;
}

/* ------------------------------------------------------ int8-stored parameters */

/* int8 storage of one stage's parameters [HARP 2.4 "deployment efficiency":
 * the parameters may be kept in int8]. The pages give no scheme; the reading
 * here is symmetric per-stage absmax: scale = max|theta| / 127 rounded to
 * float, q = clamp(rint(theta / scale), -127, 127), theta^ = scale * q. An
 * all-zero stage gets scale 0 and q = 0. */
int orc_theta_quantize(int64_t n, const double *theta, int8_t *q, float *scale)
{
    double amax = 0.0;
    for (int64_t i = 0; i < n; ++i)
        if (fabs(theta[i]) > amax) amax = fabs(theta[i]);
    if (!(amax < INFINITY)) return ORC_BAD;
    float s = (float)(amax / 127.0);
    *scale = s;
    for (int64_t i = 0; i < n; ++i) {
        double v = (s > 0.0f) ? rint(theta[i] / (double)s) : 0.0;
        if (v > 127.0) v = 127.0;
        if (v < -127.0) v = -127.0;
        q[i] = (int8_t)v;
    }
    return ORC_OK;
}

/* Blocks of one stage from int8-stored parameters [HARP 2.2]:
 * B_c = Q(theta_c) G_b. Group c holds P = b(b-1)/2 stored values, the strict
 * upper triangle of its skew-symmetric generator in row-major order
 * ((0,1), (0,2), ..., (0,b-1), (1,2), ...); theta = scale * q.
 *   b = 2: Q is the Givens rotation by the one angle theta_c.
 *   b > 2: A[i][j] = theta (i < j), -theta (i > j), 0 on the diagonal, and Q
 *          is the Cayley map (I - A)^-1 (I + A).
 *   b = 1: Q = [1].
 * G: the base mixer [b][b] (float values promoted), or NULL for the
 * normalised Sylvester matrix (b a power of two).
 * out: [n_groups][b][b] row-major (out k, in j). */
int orc_theta_blocks(int b, int64_t n_groups, const int8_t *q, double scale,
                     const double *G, double *out)
{
    if (b < 1) return ORC_BAD;
    const int64_t P = (int64_t)b * (b - 1) / 2;
    double *Gm = (double *)malloc(sizeof(double) * b * b);
    double *A = (double *)malloc(sizeof(double) * b * b);
    double *Qm = (double *)malloc(sizeof(double) * b * b);
    int st = ORC_OK;
    if (!Gm || !A || !Qm) { st = ORC_BAD; goto done; }
    if (G) memcpy(Gm, G, sizeof(double) * b * b);
    else if ((st = orc_sylvester(b, Gm)) != ORC_OK) goto done;
    for (int64_t c = 0; c < n_groups; ++c) {
        const int8_t *qc = q + c * P;
        if (b == 1) {
            Qm[0] = 1.0;
        } else if (b == 2) {
            orc_givens(scale * (double)qc[0], Qm);
        } else {
            int64_t e = 0;
            for (int i = 0; i < b; ++i) A[i * b + i] = 0.0;
            for (int i = 0; i < b; ++i)
                for (int j = i + 1; j < b; ++j, ++e) {
                    A[i * b + j] = scale * (double)qc[e];
                    A[j * b + i] = -A[i * b + j];
                }
            if ((st = orc_cayley(b, A, Qm)) != ORC_OK) goto done;
        }
        double *B = out + c * (int64_t)b * b;
        for (int i = 0; i < b; ++i)
            for (int j = 0; j < b; ++j) {
                double acc = 0.0;
                for (int k = 0; k < b; ++k) acc += Qm[i * b + k] * Gm[k * b + j];
                B[i * b + j] = acc;
            }
    }
done:
    free(Gm);
    free(A);
    free(Qm);
    return st;
}

/* ------------------------------------------------------------------ quantizer */

/* Standard normal density and distribution function. */
static double orc_phi(double z) { return exp(-0.5 * z * z) / sqrt(2.0 * M_PI); }
static double orc_Phi(double z) { return 0.5 * erfc(-z / sqrt(2.0)); }

/* Lloyd-Max centroids for N(0,1) with K = 2^bits levels [PQ 2]. Fixed point:
 * thresholds are midpoints of neighbouring centroids, and each centroid is the
 * conditional mean of its cell, E[Z | t_{k-1} < Z < t_k] =
 * (phi(t_{k-1}) - phi(t_k)) / (Phi(t_k) - Phi(t_{k-1})). Start from the
 * normal quantiles of the cell centres; iterate to a max change below 1e-15
 * (or 200000 iterations); finally make the table exactly odd-symmetric. */
int orc_lloyd_max(int bits, double *c, int *iterations)
{
    static double cache[9][256];
    static int cache_iters[9];
    static int cached[9];
    if (bits < 1 || bits > 8) return ORC_BAD;
    if (cached[bits]) {
        memcpy(c, cache[bits], sizeof(double) * (1 << bits));
        if (iterations) *iterations = cache_iters[bits];
        return ORC_OK;
    }
    int K = 1 << bits;
    double *t = (double *)malloc(sizeof(double) * (K + 1));
    if (!t) return ORC_BAD;
    for (int k = 0; k < K; ++k) {        /* quantile of (k + 1/2)/K by bisection */
        double p = (k + 0.5) / K, lo = -10.0, hi = 10.0;
        for (int it = 0; it < 200; ++it) {
            double mid = 0.5 * (lo + hi);
            if (orc_Phi(mid) < p) lo = mid; else hi = mid;
        }
        c[k] = 0.5 * (lo + hi);
    }
    int it = 0;
    for (; it < 200000; ++it) {
        t[0] = -INFINITY;
        t[K] = INFINITY;
        for (int k = 1; k < K; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
        double change = 0.0;
        for (int k = 0; k < K; ++k) {
            double pa = isinf(t[k]) ? 0.0 : orc_phi(t[k]);
            double pb = isinf(t[k + 1]) ? 0.0 : orc_phi(t[k + 1]);
            double mass = orc_Phi(t[k + 1]) - orc_Phi(t[k]);
            double nc = (pa - pb) / mass;
            double dc = fabs(nc - c[k]);
            if (dc > change) change = dc;
            c[k] = nc;
        }
        if (change < 1e-15) break;
    }
    for (int k = 0; k < K / 2; ++k) {
        double v = 0.5 * (c[K - 1 - k] - c[k]);
        c[k] = -v;
        c[K - 1 - k] = v;
    }
    if (iterations) *iterations = it;
    memcpy(cache[bits], c, sizeof(double) * K);
    cache_iters[bits] = it;
    cached[bits] = 1;
    free(t);
    return ORC_OK;
}

/* float64 -> IEEE binary16 bits, round to nearest even, saturating at the
 * largest finite value 65504 (no infinities are produced). x >= 0 only. */
uint16_t orc_f16_bits(double x)
{
    if (!(x > 0.0)) return 0;                      /* 0 (and NaN) -> +0 */
    if (x >= 65504.0) return 0x7BFF;
    int e;
    (void)frexp(x, &e);                            /* x = f 2^e, f in [0.5, 1) */
    int E = e - 1;                                  /* x = (2f) 2^E, 2f in [1, 2) */
    double q;
    if (E < -14) {                                  /* subnormal: units of 2^-24 */
        q = ldexp(x, 24);
        double r = nearbyint(q);                    /* default mode: ties to even */
        return (uint16_t)r;                         /* r == 1024 is the smallest normal */
    }
    q = ldexp(x, 10 - E);                           /* in [1024, 2048) */
    double r = nearbyint(q);
    if (r == 2048.0) { r = 1024.0; E += 1; }
    if (E > 15) return 0x7BFF;
    uint16_t bits = (uint16_t)(((E + 15) << 10) | ((int)r - 1024));
    if (bits > 0x7BFF) bits = 0x7BFF;
    return bits;
}

double orc_f16_value(uint16_t h)
{
    int e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0) v = ldexp((double)f, -24);
    else if (e == 31) v = f ? NAN : INFINITY;
    else v = ldexp((double)(f + 1024), e - 25);
    return (h & 0x8000) ? -v : v;
}

/* fp32 table the quantizer uses: centroids rounded to float, midpoints of the
 * rounded centroids computed in double and rounded to float [PQ 2: fp32
 * centroid table]. */
static void orc_tables(int bits, const double *c64, float *cent, float *thr)
{
    int K = 1 << bits;
    for (int k = 0; k < K; ++k) cent[k] = (float)c64[k];
    for (int k = 0; k + 1 < K; ++k) thr[k] = (float)(0.5 * ((double)cent[k] + (double)cent[k + 1]));
}

/* Group-wise quantisation of X [rows x cols] in float64.
 * kind 0 = Lloyd-Max (scale = RMS, codes by midpoint count),
 * kind 1 = absmax (scale = max|x| / qmax, codes = clamp(rint(x/s)) + 2^(b-1)).
 * Outputs: codes [rows x cols] (one byte each, unpacked), scales [rows x
 * cols/group] fp16 bits. Diagnostics (either may be NULL):
 *  margin[i] = distance of z = x/s to the nearest decision boundary;
 *  scale_margin[g] = |pre-rounding scale - nearest fp16 rounding midpoint|
 *                    relative to the scale (how close the fp16 decision was). */
int orc_quantize_mode(int kind, int bits, int64_t group, int scale_mode, int64_t rows, int64_t cols,
                      const double *X, uint8_t *codes, uint16_t *scales,
                      double *margin, double *scale_margin);

int orc_quantize(int kind, int bits, int64_t group, int64_t rows, int64_t cols,
                 const double *X, uint8_t *codes, uint16_t *scales,
                 double *margin, double *scale_margin)
{
    return orc_quantize_mode(kind, bits, group, 0, rows, cols, X, codes, scales, margin, scale_margin);
}

/* As orc_quantize, with the Lloyd-Max group scale chosen by scale_mode:
 *  0: s = sqrt(mean of squares) (the default reading of PolarQuant's
 *     normalisation to N(0,1));
 *  1: s = max|x| / c_{K-1}, the group's largest magnitude mapped onto the
 *     outermost fp32 centroid (the alternative kept as a flag).
 * Absmax codebooks accept mode 0 only. */
int orc_quantize_mode(int kind, int bits, int64_t group, int scale_mode, int64_t rows, int64_t cols,
                      const double *X, uint8_t *codes, uint16_t *scales,
                      double *margin, double *scale_margin)
{
    if (bits < 2 || bits > 5 || group <= 0 || cols % group) return ORC_BAD;
    if (scale_mode < 0 || scale_mode > 1 || (kind != 0 && scale_mode != 0)) return ORC_BAD;
    int K = 1 << bits;
    int qmax = (1 << (bits - 1)) - 1;
    double c64[32];
    float cent[32], thr[32];
    if (kind == 0) {
        if (orc_lloyd_max(bits, c64, NULL)) return ORC_BAD;
        orc_tables(bits, c64, cent, thr);
    }
    int64_t ng = cols / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t g = 0; g < ng; ++g) {
            const double *x = X + r * cols + g * group;
            double s_exact;
            if (kind == 0 && scale_mode == 1) {
                double mx = 0.0;
                for (int64_t i = 0; i < group; ++i) if (fabs(x[i]) > mx) mx = fabs(x[i]);
                s_exact = mx / (double)cent[K - 1];
            } else if (kind == 0) {
                double ss = 0.0;
                for (int64_t i = 0; i < group; ++i) ss += x[i] * x[i];
                s_exact = sqrt(ss / (double)group);
            } else {
                double mx = 0.0;
                for (int64_t i = 0; i < group; ++i) if (fabs(x[i]) > mx) mx = fabs(x[i]);
                s_exact = mx / (double)qmax;
            }
            uint16_t sb = orc_f16_bits(s_exact);
            double s = orc_f16_value(sb);
            scales[r * ng + g] = sb;
            if (scale_margin) {
                /* distance to the fp16 rounding boundaries around s_exact */
                double best = INFINITY;
                for (int dlt = -1; dlt <= 1; ++dlt) {
                    int nb = (int)sb + dlt;
                    if (nb < 0 || nb > 0x7BFF) continue;
                    double a = orc_f16_value((uint16_t)nb);
                    double bnext = orc_f16_value((uint16_t)(nb + 1));
                    double mid = 0.5 * (a + bnext);
                    double dd = fabs(s_exact - mid);
                    if (dd < best) best = dd;
                }
                scale_margin[r * ng + g] = (s_exact > 0.0) ? best / s_exact : INFINITY;
            }
            for (int64_t i = 0; i < group; ++i) {
                int64_t idx = r * cols + g * group + i;
                int code;
                double mrg = INFINITY;
                if (s == 0.0) {
                    code = (kind == 0) ? K / 2 : (1 << (bits - 1));
                } else {
                    double z = x[i] / s;
                    if (kind == 0) {
                        code = 0;
                        for (int k = 0; k + 1 < K; ++k) {
                            if (z > (double)thr[k]) ++code;
                            double dd = fabs(z - (double)thr[k]);
                            if (dd < mrg) mrg = dd;
                        }
                    } else {
                        double q = nearbyint(z);
                        if (q > qmax) q = qmax;
                        if (q < -qmax) q = -qmax;
                        code = (int)q + (1 << (bits - 1));
                        double fr = z - floor(z);            /* distance to n + 1/2 */
                        if (z > -qmax - 0.5 && z < qmax + 0.5) mrg = fabs(fr - 0.5);
                    }
                }
                codes[idx] = (uint8_t)code;
                if (margin) margin[idx] = mrg;
            }
        }
    return ORC_OK;
}

/* Restored weights in a 16- or 32-bit storage type [PQ 3: the Q5 weights,
 * dequantised and rotated back, are kept in fp16 and then handed to a
 * downstream INT4 absmax quantiser]. Each value is rounded to nearest even
 * from float64: kind 0 float, 1 bfloat16 (normal range), 2 fp16 (saturating
 * at +-65504, the same conversion as the scales). */
int orc_round_mid(int kind, int64_t n, const double *x, double *out)
{
    if (kind < 0 || kind > 2) return ORC_BAD;
    for (int64_t i = 0; i < n; ++i) {
        double v = x[i], a = fabs(v), r;
        if (kind == 0) {
            r = (double)(float)a;
        } else if (kind == 2) {
            r = orc_f16_value(orc_f16_bits(a));
        } else if (a == 0.0) {
            r = 0.0;
        } else {
            int e;
            (void)frexp(a, &e);                     /* a = f 2^e, f in [0.5, 1) */
            r = ldexp(nearbyint(ldexp(a, 8 - e)), e - 8);   /* 8 significant bits */
        }
        out[i] = (v < 0.0) ? -r : r;
    }
    return ORC_OK;
}

/* Dequantise: x = s * c[code] (Lloyd-Max, fp32 centroid table) or
 * x = s * (code - 2^(b-1)) (absmax). */
int orc_dequantize(int kind, int bits, int64_t group, int64_t rows, int64_t cols,
                   const uint8_t *codes, const uint16_t *scales, double *X)
{
    if (bits < 2 || bits > 5 || group <= 0 || cols % group) return ORC_BAD;
    double c64[32];
    float cent[32], thr[32];
    if (kind == 0) {
        if (orc_lloyd_max(bits, c64, NULL)) return ORC_BAD;
        orc_tables(bits, c64, cent, thr);
    }
    int64_t ng = cols / group;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < cols; ++i) {
            double s = orc_f16_value(scales[r * ng + i / group]);
            int code = codes[r * cols + i];
            X[r * cols + i] = (kind == 0) ? s * (double)cent[code]
                                          : s * (double)(code - (1 << (bits - 1)));
        }
    return ORC_OK;
}

/* LSB-first bit packing of each row: code i occupies bits [b i, b i + b). */
int orc_pack(int bits, int64_t rows, int64_t cols, const uint8_t *codes, uint8_t *packed)
{
    if ((cols * bits) % 8) return ORC_BAD;
    int64_t rb = cols * bits / 8;
    memset(packed, 0, (size_t)(rows * rb));
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < cols; ++i) {
            int v = codes[r * cols + i];
            for (int q = 0; q < bits; ++q) {
                int64_t bit = (int64_t)bits * i + q;
                if ((v >> q) & 1) packed[r * rb + bit / 8] |= (uint8_t)(1u << (bit % 8));
            }
        }
    return ORC_OK;
}

int orc_unpack(int bits, int64_t rows, int64_t cols, const uint8_t *packed, uint8_t *codes)
{
    if ((cols * bits) % 8) return ORC_BAD;
    int64_t rb = cols * bits / 8;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t i = 0; i < cols; ++i) {
            int v = 0;
            for (int q = 0; q < bits; ++q) {
                int64_t bit = (int64_t)bits * i + q;
                v |= ((packed[r * rb + bit / 8] >> (bit % 8)) & 1) << q;
            }
            codes[r * cols + i] = (uint8_t)v;
        }
    return ORC_OK;
}

/* --------------------------------------------------- sampled two-sided rows */

/* Rows `which[0..n)` of W' = M_L W M_R^T for W [rows x cols] (rows = d_L,
 * cols = d_R) without forming the whole product: row r of M_L is
 * (M_L^T e_r)^T, so (M_L W)[r, :] = sum_i (M_L^T e_r)_i W[i, :], followed by
 * the right processor on that row. Left may be absent (m_l = 0). */
int orc_two_sided_rows(int64_t rows, int64_t cols,
                       int m_l, const int32_t *radix_l, const double *blocks_l, const double *signs_l,
                       int m_r, const int32_t *radix_r, const double *blocks_r, const double *signs_r,
                       const double *W, int64_t n, const int64_t *which, double *out)
{
    double *e = (double *)calloc((size_t)rows, sizeof(double));
    double *u = (double *)malloc(sizeof(double) * rows);
    double *v = (double *)malloc(sizeof(double) * cols);
    int st = ORC_OK;
    if (!e || !u || !v) { st = ORC_BAD; goto done; }
    for (int64_t q = 0; q < n; ++q) {
        int64_t r = which[q];
        if (r < 0 || r >= rows) { st = ORC_BAD; goto done; }
        if (m_l > 0) {
            memset(e, 0, sizeof(double) * rows);
            e[r] = 1.0;
            st = orc_apply(rows, m_l, radix_l, blocks_l, signs_l, 1, e, u);
            if (st) goto done;
            memset(v, 0, sizeof(double) * cols);
            for (int64_t i = 0; i < rows; ++i) {
                double ui = u[i];
                const double *w = W + i * cols;
                for (int64_t j = 0; j < cols; ++j) v[j] += ui * w[j];
            }
        } else {
            memcpy(v, W + r * cols, sizeof(double) * cols);
        }
        st = orc_apply(cols, m_r, radix_r, blocks_r, signs_r, 0, v, out + q * cols);
        if (st) goto done;
    }
done:
    free(e);
    free(u);
    free(v);
    return st;
}

/* Rows `which` of the inverse  W = M_L^T W' M_R  for W' given in full
 * (float64): (M_L^T W')[r, :] = sum_i (M_L e_r)_i W'[i, :], then M_R^T on
 * the row. */
int orc_inverse_rows(int64_t rows, int64_t cols,
                     int m_l, const int32_t *radix_l, const double *blocks_l, const double *signs_l,
                     int m_r, const int32_t *radix_r, const double *blocks_r, const double *signs_r,
                     const double *Wp, int64_t n, const int64_t *which, double *out)
{
    double *e = (double *)calloc((size_t)rows, sizeof(double));
    double *u = (double *)malloc(sizeof(double) * rows);
    double *v = (double *)malloc(sizeof(double) * cols);
    int st = ORC_OK;
    if (!e || !u || !v) { st = ORC_BAD; goto done; }
    for (int64_t q = 0; q < n; ++q) {
        int64_t r = which[q];
        if (r < 0 || r >= rows) { st = ORC_BAD; goto done; }
        if (m_l > 0) {
            memset(e, 0, sizeof(double) * rows);
            e[r] = 1.0;
            st = orc_apply(rows, m_l, radix_l, blocks_l, signs_l, 0, e, u);
            if (st) goto done;
            memset(v, 0, sizeof(double) * cols);
            for (int64_t i = 0; i < rows; ++i) {
                double ui = u[i];
                const double *w = Wp + i * cols;
                for (int64_t j = 0; j < cols; ++j) v[j] += ui * w[j];
            }
        } else {
            memcpy(v, Wp + r * cols, sizeof(double) * cols);
        }
        st = orc_apply(cols, m_r, radix_r, blocks_r, signs_r, 1, v, out + q * cols);
        if (st) goto done;
    }
done:
    free(e);
    free(u);
    free(v);
    return st;
}
