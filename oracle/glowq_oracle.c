/*
 * glowq_oracle.c -- plain, slow, obviously-correct CPU oracle for the GlowQ
 * corrected quantised linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test-suite, the smoke check and the
 * CPU-baseline leg of the benchmark may load this library.  The product path
 * (the CUDA library and its Python binding) never calls it and shares no code
 * with it.
 *
 * Sources (the GlowQ pages):
 *   - papernotes.org, "GlowQ: Group-Shared Low-Rank Approximation for Quantized
 *     LLMs", key designs 1-4 and the experimental set-up paragraph:
 *       design 1  stacked error E_cat, one shared right factor B (Prop. 1,
 *                 Eckart-Young-Mirsky);
 *       design 2  covariance-aligned objective ||(E_cat - AB) Sx^{1/2}||_F^2
 *                 (Props. 2/3), isotropic case = plain stacked SVD;
 *       design 3  thin QR core M = R_e Sx^{1/2}, randomised SVD with
 *                 oversampling p and q power iterations, balanced split
 *                 A = U_r S_r^{1/2}, B = S_r^{1/2} V_r^T lifted back with the
 *                 pseudo-inverse;
 *       design 4  R = X B_shared^T computed once per input-sharing group,
 *                 y_i = W_i^(q) X + A_i R; solo modules inline; GlowQ-S top-k
 *                 by an importance score (g_ner(u) = ||E_u||_F^2 / ||W_u||_F^2
 *                 or the GSVD energy capture g_ec, composed in the Python
 *                 layer from the QR and SVD below) with layer-order fallback
 *                 when the signal is weak;
 *       set-up    W4A16, INT4 weights with group size 128, fp16 activations,
 *                 rank 64.
 *   - thelatestinai.com, GlowQ page: Table 6 (notation and shapes),
 *     Table 11 caption (exact SVD vs Halko randomised SVD on the core M),
 *     Table 12 (p = 16 with q = 2 as the fixed values of the sweeps),
 *     Table 13 (MXFP4 / NVFP4 base weights) and Tables 14-15 (W4A8): the
 *     formats are not defined there; the sections at the end of this file
 *     state the readings taken.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - the INT4 quantiser is asymmetric round-to-nearest per (row, 128-group):
 *     mn = min(min w, 0), mx = max(max w, 0), s = fp16(fp32((mx-mn)/15)),
 *     z = clamp(rint(-mn/s), 0, 15), q = clamp(rint(w/s) + z, 0, 15), all in
 *     IEEE fp32 round-to-nearest-even with no fused multiply-add;
 *     s == 0 -> 1.0, s == inf -> 65504;
 *   - dequantisation is w_hat = fp16_RN((q - z) * s): one rounding of the
 *     exact product;
 *   - packing: code k of a row sits in nibble (k mod 8) of word k/8, lowest
 *     nibble first; zeros are one byte each;
 *   - the forward is evaluated in float64 from the exact fp16 values of X, B
 *     and A; R is not rounded.
 *
 * Parity pins for every function live in tests/test_oracle_*.py.
 *
 * Threads: the forward functions split independent outputs (tokens of R,
 * rows of Y, samples) across OpenMP threads; each output is still one
 * sequential float64 sum in k order, so the result does not depend on the
 * thread count.  ora_set_threads() fixes the count (1 = single-threaded).
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fno-fast-math -fPIC -shared.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE binary16 conversions                                                 */
/* ------------------------------------------------------------------------ */

/* Exact value of a binary16 bit pattern. */
double ora_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0x1f) {
        v = f ? NAN : INFINITY;
    } else if (e == 0) {
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-24 */
    } else {
        v = ldexp((double)(1024 + f), e - 25);   /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* Round a double to the nearest binary16 value, ties to even, in one step. */
uint16_t ora_f64_to_f16(double v)
{
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    if (isnan(v)) return (uint16_t)(sign | 0x7e00);
    if (isinf(a)) return (uint16_t)(sign | 0x7c00);
    if (a == 0.0) return sign;
    int E;
    frexp(a, &E);            /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;           /* a = (2f) * 2^e, 2f in [1, 2) */
    if (e < -14) {
        /* subnormal range: quantum 2^-24.  A result of 1024 is the smallest
           normal number, whose bit pattern is exactly 1024. */
        double m = nearbyint(ldexp(a, 24));
        return (uint16_t)(sign | (uint16_t)m);
    }
    if (e > 15) return (uint16_t)(sign | 0x7c00);
    /* normal range: 11 significant bits, quantum 2^(e-10) */
    double m = nearbyint(ldexp(a, 10 - e));   /* in [1024, 2048] */
    long bits = ((long)(e + 15) << 10) + ((long)m - 1024);  /* carry ok */
    if (bits >= 0x7c00) return (uint16_t)(sign | 0x7c00);
    return (uint16_t)(sign | (uint16_t)bits);
}

uint16_t ora_f32_to_f16(float v) { return ora_f64_to_f16((double)v); }

/* ------------------------------------------------------------------------ */
/* INT4 g128 asymmetric quantisation (set-up paragraph: INT4, group 128)     */
/* ------------------------------------------------------------------------ */

static float clamp_code(float v)
{
    if (!(v >= 0.0f)) v = 0.0f;   /* also maps NaN to 0 */
    if (v > 15.0f) v = 15.0f;
    return v;
}

/*
 * W: O x d fp32 row-major.  Outputs: q [O][d/8] uint32, s [O][d/gs] fp16
 * bits, z [O][d/gs] uint8.  Returns 0, or -1 on bad sizes.
 */
int ora_quantize_int4(const float* W, int64_t O, int64_t d, int32_t gs,
                      uint32_t* q, uint16_t* s, uint8_t* z)
{
    if (O < 0 || d < 0 || gs <= 0 || gs % 8 != 0 || d % gs != 0) return -1;
    int64_t ng = d / gs;
    memset(q, 0, (size_t)(O * (d / 8)) * sizeof(uint32_t));
    for (int64_t o = 0; o < O; ++o) {
        for (int64_t g = 0; g < ng; ++g) {
            const float* w = W + o * d + g * gs;
            volatile float mn = 0.0f, mx = 0.0f;
            for (int k = 0; k < gs; ++k) {
                if (w[k] < mn) mn = w[k];
                if (w[k] > mx) mx = w[k];
            }
            volatile float range = mx - mn;
            volatile float s32 = range / 15.0f;
            uint16_t sh = ora_f32_to_f16(s32);
            if ((sh & 0x7fff) == 0) sh = 0x3c00;          /* 1.0 */
            if ((sh & 0x7fff) == 0x7c00) sh = 0x7bff;     /* 65504 */
            float sf = (float)ora_f16_to_f64(sh);
            volatile float zq = -mn / sf;
            float zf = clamp_code(rintf(zq));
            s[o * ng + g] = sh;
            z[o * ng + g] = (uint8_t)zf;
            for (int k = 0; k < gs; ++k) {
                volatile float t = w[k] / sf;
                float c = clamp_code(rintf(t) + zf);
                int64_t col = g * gs + k;
                q[o * (d / 8) + col / 8] |= ((uint32_t)c & 0xfu) << (4 * (col % 8));
            }
        }
    }
    return 0;
}

/* code of row o, column k */
static inline int code_at(const uint32_t* q, int64_t d, int64_t o, int64_t k)
{
    return (int)((q[o * (d / 8) + k / 8] >> (4 * (k % 8))) & 0xfu);
}

/* Unpack codes only: out [O][d] uint8. */
int ora_unpack_int4(const uint32_t* q, int64_t O, int64_t d, uint8_t* codes)
{
    if (O < 0 || d < 0 || d % 8 != 0) return -1;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t k = 0; k < d; ++k)
            codes[o * d + k] = (uint8_t)code_at(q, d, o, k);
    return 0;
}

/* w_hat = fp16_RN((q - z) * s), the product taken exactly. out: [O][d] fp16 bits. */
int ora_dequant_int4(const uint32_t* q, const uint16_t* s, const uint8_t* z,
                     int64_t O, int64_t d, int32_t gs, uint16_t* out)
{
    if (O < 0 || d < 0 || gs <= 0 || d % gs != 0 || d % 8 != 0) return -1;
    int64_t ng = d / gs;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t k = 0; k < d; ++k) {
            int64_t g = k / gs;
            double prod = (double)(code_at(q, d, o, k) - (int)z[o * ng + g]) *
                          ora_f16_to_f64(s[o * ng + g]);
            out[o * d + k] = ora_f64_to_f16(prod);
        }
    return 0;
}

/* E = W - w_hat in float64, and the squared Frobenius norms used by g_ner. */
int ora_quant_error(const float* W, const uint32_t* q, const uint16_t* s,
                    const uint8_t* z, int64_t O, int64_t d, int32_t gs,
                    double* E, double* err_fro2, double* w_fro2)
{
    if (O < 0 || d < 0 || gs <= 0 || d % gs != 0) return -1;
    int64_t ng = d / gs;
    double se = 0.0, sw = 0.0;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t k = 0; k < d; ++k) {
            int64_t g = k / gs;
            double what = ora_f16_to_f64(ora_f64_to_f16(
                (double)(code_at(q, d, o, k) - (int)z[o * ng + g]) *
                ora_f16_to_f64(s[o * ng + g])));
            double w = (double)W[o * d + k];
            double e = w - what;
            if (E) E[o * d + k] = e;
            se += e * e;
            sw += w * w;
        }
    if (err_fro2) *err_fro2 = se;
    if (w_fro2) *w_fro2 = sw;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Forward: R = X B^T once per group; y_i = X w_hat_i^T + R A_i^T            */
/* (key design 4; solo modules compute their own R inline)                   */
/* ------------------------------------------------------------------------ */

/* R[t][j] = sum_k X[t][k] B[j][k]   (X: T x d fp16, B: r x d fp16) */
int ora_anchor_project(const uint16_t* X, const uint16_t* B, int64_t T,
                       int64_t d, int32_t r, double* R)
{
    if (T < 0 || d < 0 || r < 0) return -1;
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int32_t j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < d; ++k)
                acc += ora_f16_to_f64(X[t * d + k]) * ora_f16_to_f64(B[(int64_t)j * d + k]);
            R[t * r + j] = acc;
        }
    return 0;
}

/*
 * One module given the group's R:
 *   Y[t][o] = sum_k X[t][k] w_hat[o][k] + sum_j R[t][j] A[o][j]
 * A may be NULL (or r == 0): the correction is disabled (GlowQ-S off unit).
 * Y: T x O float64, row-major (token-major).
 */
int ora_module_forward(const uint32_t* q, const uint16_t* s, const uint8_t* z,
                       int64_t O, int64_t d, int32_t gs, const uint16_t* A,
                       int32_t r, const double* R, const uint16_t* X, int64_t T,
                       double* Y)
{
    if (O < 0 || d < 0 || T < 0 || gs <= 0 || d % gs != 0) return -1;
    double* xd = (double*)malloc((size_t)(T * d > 0 ? T * d : 1) * sizeof(double));
    if (!xd) return -2;
    for (int64_t i = 0; i < T * d; ++i) xd[i] = ora_f16_to_f64(X[i]);
    int64_t ng = d / gs;
    int failed = 0;
#pragma omp parallel
    {
        /* one dequantised row per thread */
        double* whd = (double*)malloc((size_t)(d > 0 ? d : 1) * sizeof(double));
        if (!whd) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(static)
        for (int64_t o = 0; o < O; ++o) {
            if (!whd) continue;
            for (int64_t k = 0; k < d; ++k) {
                int64_t g = k / gs;
                double prod = (double)(code_at(q, d, o, k) - (int)z[o * ng + g]) *
                              ora_f16_to_f64(s[o * ng + g]);
                whd[k] = ora_f16_to_f64(ora_f64_to_f16(prod));
            }
            for (int64_t t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int64_t k = 0; k < d; ++k)
                    acc += xd[t * d + k] * whd[k];
                if (A && r > 0 && R)
                    for (int32_t j = 0; j < r; ++j)
                        acc += R[t * r + j] * ora_f16_to_f64(A[o * r + j]);
                Y[t * O + o] = acc;
            }
        }
        free(whd);
    }
    free(xd);
    return failed ? -2 : 0;
}

/* Solo module: its own R = X B^T computed inline, nothing shared. */
int ora_solo_forward(const uint32_t* q, const uint16_t* s, const uint8_t* z,
                     int64_t O, int64_t d, int32_t gs, const uint16_t* A,
                     const uint16_t* B, int32_t r, const uint16_t* X, int64_t T,
                     double* Y)
{
    double* R = NULL;
    int use = (A && B && r > 0);
    if (use) {
        R = (double*)malloc((size_t)(T * r > 0 ? T * r : 1) * sizeof(double));
        if (!R) return -2;
        ora_anchor_project(X, B, T, d, r, R);
    }
    int rc = ora_module_forward(q, s, z, O, d, gs, use ? A : NULL, use ? r : 0, R, X, T, Y);
    free(R);
    return rc;
}

/*
 * Sampled outputs: out[i] = Y[t_idx[i]][o_idx[i]] of one module, for checks
 * at sizes where the full product is too slow on the CPU.
 */
int ora_module_forward_sampled(const uint32_t* q, const uint16_t* s, const uint8_t* z,
                               int64_t O, int64_t d, int32_t gs, const uint16_t* A,
                               const uint16_t* B, int32_t r, const uint16_t* X, int64_t T,
                               int64_t n, const int64_t* t_idx, const int64_t* o_idx,
                               double* out)
{
    if (gs <= 0 || d % gs != 0) return -1;
    int64_t ng = d / gs;
    for (int64_t i = 0; i < n; ++i)
        if (t_idx[i] < 0 || t_idx[i] >= T || o_idx[i] < 0 || o_idx[i] >= O) return -1;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t i = 0; i < n; ++i) {
        int64_t t = t_idx[i], o = o_idx[i];
        double acc = 0.0;
        for (int64_t k = 0; k < d; ++k) {
            int64_t g = k / gs;
            double prod = (double)(code_at(q, d, o, k) - (int)z[o * ng + g]) *
                          ora_f16_to_f64(s[o * ng + g]);
            acc += ora_f16_to_f64(X[t * d + k]) * ora_f16_to_f64(ora_f64_to_f16(prod));
        }
        if (A && B && r > 0) {
            for (int32_t j = 0; j < r; ++j) {
                double rj = 0.0;
                for (int64_t k = 0; k < d; ++k)
                    rj += ora_f16_to_f64(X[t * d + k]) * ora_f16_to_f64(B[(int64_t)j * d + k]);
                acc += rj * ora_f16_to_f64(A[o * r + j]);
            }
        }
        out[i] = acc;
    }
    return 0;
}

/* Thread count of the OpenMP loops (n >= 1); returns the count in effect. */
int ora_set_threads(int32_t n)
{
    if (n >= 1) omp_set_num_threads(n);
    return omp_get_max_threads();
}

/* ------------------------------------------------------------------------ */
/* Dense linear algebra for the offline group solve (key design 3)           */
/* ------------------------------------------------------------------------ */

/* C (m x n) = A (m x k) * B (k x n), all row-major; ta/tb transpose flags. */
static void matmul(const double* A, const double* B, double* C, int64_t m,
                   int64_t n, int64_t k, int ta, int tb)
{
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t l = 0; l < k; ++l) {
                double a = ta ? A[l * m + i] : A[i * k + l];
                double b = tb ? B[j * k + l] : B[l * n + j];
                acc += a * b;
            }
            C[i * n + j] = acc;
        }
}

int ora_matmul(const double* A, const double* B, double* C, int64_t m,
               int64_t n, int64_t k, int32_t ta, int32_t tb)
{
    matmul(A, B, C, m, n, k, ta, tb);
    return 0;
}

/*
 * Householder thin QR of A (m x n, row-major): A = Q R with Q m x kk having
 * orthonormal columns and R kk x n upper trapezoidal, kk = min(m, n).
 */
int ora_householder_qr(const double* A, int64_t m, int64_t n, double* Q, double* R)
{
    int64_t kk = m < n ? m : n;
    double* W = (double*)malloc((size_t)(m * n > 0 ? m * n : 1) * sizeof(double));
    double* V = (double*)malloc((size_t)(m * (kk > 0 ? kk : 1)) * sizeof(double) + 8);
    double* beta = (double*)malloc((size_t)(kk > 0 ? kk : 1) * sizeof(double));
    if (!W || !V || !beta) { free(W); free(V); free(beta); return -2; }
    memcpy(W, A, (size_t)(m * n) * sizeof(double));
    for (int64_t j = 0; j < kk; ++j) {
        /* reflector for column j, rows j..m-1 */
        double norm = 0.0;
        for (int64_t i = j; i < m; ++i) norm += W[i * n + j] * W[i * n + j];
        norm = sqrt(norm);
        double* v = V + j * m;
        for (int64_t i = 0; i < m; ++i) v[i] = 0.0;
        if (norm == 0.0) { beta[j] = 0.0; continue; }
        double x0 = W[j * n + j];
        double alpha = x0 >= 0 ? -norm : norm;      /* avoid cancellation */
        for (int64_t i = j; i < m; ++i) v[i] = W[i * n + j];
        v[j] = x0 - alpha;
        double vnorm2 = 0.0;
        for (int64_t i = j; i < m; ++i) vnorm2 += v[i] * v[i];
        beta[j] = vnorm2 > 0 ? 2.0 / vnorm2 : 0.0;
        /* W <- (I - beta v v^T) W on columns j..n-1 */
        for (int64_t c = j; c < n; ++c) {
            double dot = 0.0;
            for (int64_t i = j; i < m; ++i) dot += v[i] * W[i * n + c];
            dot *= beta[j];
            for (int64_t i = j; i < m; ++i) W[i * n + c] -= dot * v[i];
        }
    }
    /* R = first kk rows of W, zero below the diagonal */
    for (int64_t i = 0; i < kk; ++i)
        for (int64_t c = 0; c < n; ++c)
            R[i * n + c] = (c < i) ? 0.0 : W[i * n + c];
    /* Q = H_0 H_1 ... H_{kk-1} applied to the first kk columns of I */
    for (int64_t i = 0; i < m; ++i)
        for (int64_t c = 0; c < kk; ++c) Q[i * kk + c] = (i == c) ? 1.0 : 0.0;
    for (int64_t j = kk - 1; j >= 0; --j) {
        double* v = V + j * m;
        if (beta[j] == 0.0) continue;
        for (int64_t c = 0; c < kk; ++c) {
            double dot = 0.0;
            for (int64_t i = j; i < m; ++i) dot += v[i] * Q[i * kk + c];
            dot *= beta[j];
            for (int64_t i = j; i < m; ++i) Q[i * kk + c] -= dot * v[i];
        }
    }
    free(W);
    free(V);
    free(beta);
    return 0;
}

/*
 * One-sided Jacobi (Hestenes) SVD of A (m x n, row-major): A = U diag(S) V^T,
 * kk = min(m, n) triplets sorted by descending S.  U m x kk, V n x kk.
 * Works on A if m >= n, else on A^T (and swaps the roles of U and V).
 */
int ora_jacobi_svd(const double* A, int64_t m, int64_t n, double* U, double* S, double* V)
{
    int tr = m < n;
    int64_t rows = tr ? n : m, cols = tr ? m : n;   /* rows >= cols */
    double* G = (double*)malloc((size_t)(rows * cols > 0 ? rows * cols : 1) * sizeof(double));
    double* J = (double*)malloc((size_t)(cols * cols > 0 ? cols * cols : 1) * sizeof(double));
    if (!G || !J) { free(G); free(J); return -2; }
    /* G column-major-ish: G[c*rows + i] = column c, row i */
    for (int64_t i = 0; i < rows; ++i)
        for (int64_t c = 0; c < cols; ++c)
            G[c * rows + i] = tr ? A[c * n + i] : A[i * n + c];
    for (int64_t a = 0; a < cols; ++a)
        for (int64_t b = 0; b < cols; ++b) J[a * cols + b] = (a == b) ? 1.0 : 0.0;
    const double eps = 1e-15;
    for (int sweep = 0; sweep < 80; ++sweep) {
        int rotated = 0;
        for (int64_t p = 0; p < cols - 1; ++p)
            for (int64_t q = p + 1; q < cols; ++q) {
                double* gp = G + p * rows;
                double* gq = G + q * rows;
                double alpha = 0, beta = 0, gamma = 0;
                for (int64_t i = 0; i < rows; ++i) {
                    alpha += gp[i] * gp[i];
                    beta += gq[i] * gq[i];
                    gamma += gp[i] * gq[i];
                }
                if (gamma == 0.0 || fabs(gamma) <= eps * sqrt(alpha * beta)) continue;
                rotated = 1;
                double zeta = (beta - alpha) / (2.0 * gamma);
                double t = (zeta >= 0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                double c = 1.0 / sqrt(1.0 + t * t), sn = c * t;
                for (int64_t i = 0; i < rows; ++i) {
                    double x = gp[i], y = gq[i];
                    gp[i] = c * x - sn * y;
                    gq[i] = sn * x + c * y;
                }
                double* jp = J + p * cols;   /* J stored column-wise as well */
                double* jq = J + q * cols;
                for (int64_t i = 0; i < cols; ++i) {
                    double x = jp[i], y = jq[i];
                    jp[i] = c * x - sn * y;
                    jq[i] = sn * x + c * y;
                }
            }
        if (!rotated) break;
    }
    /* singular values = column norms; sort descending */
    int64_t* idx = (int64_t*)malloc((size_t)(cols > 0 ? cols : 1) * sizeof(int64_t));
    double* nrm = (double*)malloc((size_t)(cols > 0 ? cols : 1) * sizeof(double));
    for (int64_t c = 0; c < cols; ++c) {
        double acc = 0;
        for (int64_t i = 0; i < rows; ++i) acc += G[c * rows + i] * G[c * rows + i];
        nrm[c] = sqrt(acc);
        idx[c] = c;
    }
    for (int64_t a = 1; a < cols; ++a) {          /* insertion sort, stable */
        int64_t key = idx[a];
        int64_t b = a - 1;
        while (b >= 0 && nrm[idx[b]] < nrm[key]) { idx[b + 1] = idx[b]; --b; }
        idx[b + 1] = key;
    }
    /* left vectors of the worked matrix: G columns / norm; right: J columns */
    double* Lm = tr ? V : U;    /* rows x cols */
    double* Rm = tr ? U : V;    /* cols x cols */
    for (int64_t c = 0; c < cols; ++c) {
        int64_t src = idx[c];
        double sv = nrm[src];
        S[c] = sv;
        for (int64_t i = 0; i < rows; ++i)
            Lm[i * cols + c] = sv > 0 ? G[src * rows + i] / sv : 0.0;
        for (int64_t i = 0; i < cols; ++i)
            Rm[i * cols + c] = J[src * cols + i];
    }
    /* columns of zero singular value: complete to an orthonormal set via
       Gram-Schmidt against the unit vectors (only reached for rank-deficient
       inputs; keeps U orthonormal) */
    for (int64_t c = 0; c < cols; ++c) {
        if (S[c] > 0) continue;
        for (int64_t e = 0; e < rows; ++e) {
            double* col = (double*)malloc((size_t)rows * sizeof(double));
            for (int64_t i = 0; i < rows; ++i) col[i] = (i == e) ? 1.0 : 0.0;
            for (int64_t pass = 0; pass < 2; ++pass)
                for (int64_t c2 = 0; c2 < cols; ++c2) {
                    if (c2 == c || (S[c2] == 0 && c2 > c)) continue;
                    double dot = 0;
                    for (int64_t i = 0; i < rows; ++i) dot += col[i] * Lm[i * cols + c2];
                    for (int64_t i = 0; i < rows; ++i) col[i] -= dot * Lm[i * cols + c2];
                }
            double nn = 0;
            for (int64_t i = 0; i < rows; ++i) nn += col[i] * col[i];
            nn = sqrt(nn);
            if (nn > 1e-6) {
                for (int64_t i = 0; i < rows; ++i) Lm[i * cols + c] = col[i] / nn;
                free(col);
                break;
            }
            free(col);
        }
    }
    free(idx);
    free(nrm);
    free(G);
    free(J);
    return 0;
}

/*
 * Halko randomised SVD of M (m x n) at rank `rank` with oversampling p and q
 * power iterations (Table 11 caption; Table 12 fixes p = 16, q = 2 in its
 * sweeps).  Omega (n x (rank+p)) is the Gaussian test matrix, drawn by the
 * caller.  Outputs the top `rank` triplets: U m x rank, S rank, V n x rank.
 * Each power step re-orthonormalises with a thin QR.
 */
int ora_rsvd(const double* M, int64_t m, int64_t n, int32_t rank, int32_t p,
             int32_t q, const double* Omega, double* U, double* S, double* V)
{
    int64_t l = rank + p;
    if (rank <= 0 || l > (m < n ? m : n)) return -1;
    double* Y = (double*)malloc((size_t)(m * l) * sizeof(double));
    double* Qy = (double*)malloc((size_t)(m * l) * sizeof(double));
    double* Z = (double*)malloc((size_t)(n * l) * sizeof(double));
    double* Qz = (double*)malloc((size_t)(n * l) * sizeof(double));
    double* Rt = (double*)malloc((size_t)(l * (m > n ? m : n)) * sizeof(double));
    double* Bs = (double*)malloc((size_t)(l * n) * sizeof(double));
    double* Ub = (double*)malloc((size_t)(l * l) * sizeof(double));
    double* Sb = (double*)malloc((size_t)l * sizeof(double));
    double* Vb = (double*)malloc((size_t)(n * l) * sizeof(double));
    if (!Y || !Qy || !Z || !Qz || !Rt || !Bs || !Ub || !Sb || !Vb) return -2;
    matmul(M, Omega, Y, m, l, n, 0, 0);                 /* Y = M Omega */
    ora_householder_qr(Y, m, l, Qy, Rt);
    for (int32_t it = 0; it < q; ++it) {
        matmul(M, Qy, Z, n, l, m, 1, 0);                /* Z = M^T Qy */
        ora_householder_qr(Z, n, l, Qz, Rt);
        matmul(M, Qz, Y, m, l, n, 0, 0);                /* Y = M Qz */
        ora_householder_qr(Y, m, l, Qy, Rt);
    }
    matmul(Qy, M, Bs, l, n, m, 1, 0);                   /* Bs = Qy^T M (l x n) */
    ora_jacobi_svd(Bs, l, n, Ub, Sb, Vb);               /* Bs = Ub Sb Vb^T */
    /* U = Qy Ub (top rank columns) */
    for (int64_t i = 0; i < m; ++i)
        for (int32_t c = 0; c < rank; ++c) {
            double acc = 0;
            for (int64_t a = 0; a < l; ++a) acc += Qy[i * l + a] * Ub[a * l + c];
            U[i * rank + c] = acc;
        }
    for (int32_t c = 0; c < rank; ++c) S[c] = Sb[c];
    for (int64_t i = 0; i < n; ++i)
        for (int32_t c = 0; c < rank; ++c) V[i * rank + c] = Vb[i * l + c];
    free(Y); free(Qy); free(Z); free(Qz); free(Rt); free(Bs); free(Ub); free(Sb); free(Vb);
    return 0;
}

/*
 * Whitened group solve (key designs 2 and 3).
 *   E_cat  m x d stacked error [E_1; ...; E_k]
 *   Sh     d x d  Sx^{1/2}   (symmetric PSD)
 *   Shp    d x d  pseudo-inverse of Sx^{1/2}
 *   Omega  d x (r+p) Gaussian test matrix, or NULL for the exact SVD of M.
 * Steps: E_cat = Q_e R_e (thin QR); M = R_e Sh; rank-r SVD M ~ U S V^T;
 * A = Q_e U S^{1/2} (m x r); B = S^{1/2} V^T Shp (r x d).
 * sing (r) receives the singular values of M.
 */
int ora_group_solve(const double* E_cat, int64_t m, int64_t d, const double* Sh,
                    const double* Shp, int32_t r, int32_t p, int32_t q,
                    const double* Omega, double* A, double* B, double* sing)
{
    int64_t kk = m < d ? m : d;
    if (r <= 0 || r > kk) return -1;
    double* Qe = (double*)malloc((size_t)(m * kk) * sizeof(double));
    double* Re = (double*)malloc((size_t)(kk * d) * sizeof(double));
    double* Mc = (double*)malloc((size_t)(kk * d) * sizeof(double));
    double* Uc = (double*)malloc((size_t)(kk * kk) * sizeof(double));
    double* Sc = (double*)malloc((size_t)kk * sizeof(double));
    double* Vc = (double*)malloc((size_t)(d * kk) * sizeof(double));
    double* Bw = (double*)malloc((size_t)(r * d) * sizeof(double));
    if (!Qe || !Re || !Mc || !Uc || !Sc || !Vc || !Bw) return -2;
    ora_householder_qr(E_cat, m, d, Qe, Re);
    matmul(Re, Sh, Mc, kk, d, d, 0, 0);                  /* M = R_e Sx^{1/2} */
    int64_t ucols, vcols;
    if (Omega) {
        int rc = ora_rsvd(Mc, kk, d, r, p, q, Omega, Uc, Sc, Vc);
        if (rc) return rc;
        ucols = r; vcols = r;
    } else {
        ora_jacobi_svd(Mc, kk, d, Uc, Sc, Vc);
        ucols = kk; vcols = kk;
    }
    /* A = Q_e U_r S_r^{1/2} */
    for (int64_t i = 0; i < m; ++i)
        for (int32_t c = 0; c < r; ++c) {
            double acc = 0;
            for (int64_t a = 0; a < kk; ++a) acc += Qe[i * kk + a] * Uc[a * ucols + c];
            A[i * r + c] = acc * sqrt(Sc[c]);
        }
    /* B = S_r^{1/2} V_r^T Sx^{+1/2} */
    for (int32_t c = 0; c < r; ++c)
        for (int64_t k = 0; k < d; ++k) Bw[c * d + k] = sqrt(Sc[c]) * Vc[k * vcols + c];
    matmul(Bw, Shp, B, r, d, d, 0, 0);
    for (int32_t c = 0; c < r; ++c) sing[c] = Sc[c];
    free(Qe); free(Re); free(Mc); free(Uc); free(Sc); free(Vc); free(Bw);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* GlowQ-S selective restore (key design 4)                                  */
/* ------------------------------------------------------------------------ */

/*
 * Score g_ner(u) = err_fro2[u] / w_fro2[u]; restore the top k units.
 * Ordering: descending score; exact ties by ascending (layer, kind, index).
 * Weak-signal fallback (reading): if any score is NaN, or all scores lie
 * within a relative spread of 1e-6 of the largest magnitude, the order is the
 * plain layer order (ascending layer, kind, index).
 * order[0..n-1] receives the ranking; mask[u] = 1 for the first k units.
 * Returns 1 when the fallback was taken, 0 otherwise, -1 on bad arguments.
 */
static const double* g_sc;
static const int32_t* g_layer;
static const int32_t* g_kind;
static int g_by_score;

static int unit_cmp(const void* pa, const void* pb)
{
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    if (g_by_score) {
        if (g_sc[a] > g_sc[b]) return -1;
        if (g_sc[a] < g_sc[b]) return 1;
    }
    if (g_layer[a] != g_layer[b]) return g_layer[a] < g_layer[b] ? -1 : 1;
    if (g_kind[a] != g_kind[b]) return g_kind[a] < g_kind[b] ? -1 : 1;
    return a < b ? -1 : (a > b);
}

/*
 * Rank units by an arbitrary importance score (the pages name two: the GSVD
 * energy capture g_ec and the normalised error ratio g_ner) with the same
 * tie-break and weak-signal fallback as above; restore the top k.
 * Returns 1 when the fallback was taken, 0 otherwise, -1 on bad arguments.
 */
int ora_select_by_score(const double* sc, const int32_t* layer, const int32_t* kind,
                        int32_t n, int32_t k, uint8_t* mask, int32_t* order)
{
    if (n < 0 || k < 0 || k > n) return -1;
    int any_nan = 0;
    double mx = -INFINITY, mn = INFINITY;
    for (int32_t u = 0; u < n; ++u) {
        if (isnan(sc[u])) any_nan = 1;
        else {
            if (sc[u] > mx) mx = sc[u];
            if (sc[u] < mn) mn = sc[u];
        }
    }
    int weak = any_nan || n == 0 || (mx - mn) <= 1e-6 * fmax(fabs(mx), 1e-300);
    for (int32_t u = 0; u < n; ++u) order[u] = u;
    g_sc = sc; g_layer = layer; g_kind = kind; g_by_score = !weak;
    qsort(order, (size_t)n, sizeof(int32_t), unit_cmp);
    for (int32_t u = 0; u < n; ++u) mask[u] = 0;
    for (int32_t i = 0; i < k; ++i) mask[order[i]] = 1;
    return weak ? 1 : 0;
}

int ora_select_restore(const double* err_fro2, const double* w_fro2,
                       const int32_t* layer, const int32_t* kind, int32_t n,
                       int32_t k, uint8_t* mask, int32_t* order, double* score)
{
    if (n < 0 || k < 0 || k > n) return -1;
    double* sc = (double*)malloc((size_t)(n > 0 ? n : 1) * sizeof(double));
    for (int32_t u = 0; u < n; ++u) {
        sc[u] = err_fro2[u] / w_fro2[u];
        if (score) score[u] = sc[u];
    }
    int rc = ora_select_by_score(sc, layer, kind, n, k, mask, order);
    free(sc);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Narrow floating-point base weights (thelatestinai.com GlowQ page, Table  */
/* 13: MXFP4 and NVFP4 as alternative base datatypes under GlowQ).          */
/* ------------------------------------------------------------------------ */

/*
 * The pages report only perplexities for these datatypes; the formats are
 * taken from their public definitions, and every choice below is a reading:
 *   - E2M1 element (4 bits): sign bit 3, exponent bits 2..1 with bias 1,
 *     mantissa bit 0; exponent 0 is subnormal (value m * 0.5).  Magnitudes
 *     0, 0.5, 1, 1.5, 2, 3, 4, 6.  Encoding: nearest magnitude, ties to the
 *     code whose mantissa bit is 0, saturation to 6; zero and NaN give code 0.
 *   - E4M3 (FN) scale: sign, 4 exponent bits with bias 7, 3 mantissa bits, no
 *     infinity, largest finite 448; round to nearest even, saturating at 448
 *     (a reading: some converters return NaN on overflow instead).
 *   - E8M0 scale: value 2^(e - 127) for e in 0..254.
 *   - MXFP4: blocks of 32 consecutive k of one row; shared scale
 *     X = 2^(floor(log2(amax)) - 2) (2 = the largest E2M1 exponent), E8M0
 *     code clamped to 0..254, X = 2^-127 for an all-zero block; elements
 *     E2M1(w / X) (so |w / X| in [6, 8) saturates to 6).
 *   - NVFP4: blocks of 16; one fp32 tensor scale
 *     s_t = amax_tensor / (6 * 448) (1 for an all-zero tensor); block scale
 *     S = E4M3(amax_block / (6 * s_t)); elements E2M1(w / (dec(S) * s_t)),
 *     zero when dec(S) == 0.  Scale arithmetic in IEEE fp32, no fused
 *     multiply-add, like the INT4 quantiser.
 *   - packing: two codes per byte, even k in the low nibble; one scale byte
 *     per block, row-major [O][d / block].
 *   - the W4A16 operand is w_hat = fp16_RN(exact dequantised value), one
 *     rounding, as for INT4.
 */

double ora_e2m1_decode(uint8_t c)
{
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

uint8_t ora_e2m1_encode(float v)
{
    if (!(v == v) || v == 0.0f) return 0;
    double a = fabs((double)v);
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 8; ++c) {                     /* non-negative codes */
        double dlt = fabs(a - ora_e2m1_decode((uint8_t)c));
        if (dlt < bestd || (dlt == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            bestd = dlt;
            best = c;
        }
    }
    if (a > 6.0) best = 7;                            /* saturate */
    if (best == 0) return 0;
    return (uint8_t)(best | (v < 0.0f ? 8 : 0));
}

double ora_e4m3_decode(uint8_t c)
{
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

uint8_t ora_e4m3_encode(float v)
{
    if (!(v == v)) return 0x7f;
    double a = fabs((double)v);
    int sign = v < 0.0f ? 0x80 : 0;
    if (a >= 448.0) return (uint8_t)(sign | 0x7e);     /* saturate to 448 */
    /* nearest of the 127 finite non-negative codes, ties to even mantissa */
    int best = 0;
    double bestd = INFINITY;
    for (int c = 0; c < 0x7f; ++c) {
        double dlt = fabs(a - ora_e4m3_decode((uint8_t)c));
        if (dlt < bestd || (dlt == bestd && (c & 1) == 0 && (best & 1) == 1)) {
            bestd = dlt;
            best = c;
        }
    }
    return (uint8_t)(best == 0 ? 0 : (sign | best));
}

double ora_e8m0_decode(uint8_t e) { return e == 255 ? NAN : ldexp(1.0, (int)e - 127); }

/* codes [O][d/2] (even k low nibble), scales [O][d/32] E8M0.  Returns 0 or -1. */
int ora_quantize_mxfp4(const float* W, int64_t O, int64_t d, uint8_t* codes, uint8_t* scales)
{
    if (O < 0 || d < 0 || d % 32 != 0) return -1;
    memset(codes, 0, (size_t)(O * (d / 2)));
    for (int64_t o = 0; o < O; ++o)
        for (int64_t b = 0; b < d / 32; ++b) {
            const float* w = W + o * d + b * 32;
            float amax = 0.0f;
            for (int k = 0; k < 32; ++k)
                if (fabsf(w[k]) > amax) amax = fabsf(w[k]);   /* NaN never compares greater */
            int e = 0;                                          /* E8M0 code */
            if (amax > 0.0f) {
                int ex;
                frexpf(amax, &ex);                               /* amax = f * 2^ex, f in [0.5, 1) */
                e = (ex - 1) - 2 + 127;                          /* floor(log2 amax) - 2, biased */
                if (e < 0) e = 0;
                if (e > 254) e = 254;
            }
            scales[o * (d / 32) + b] = (uint8_t)e;
            const float X = (float)ora_e8m0_decode((uint8_t)e);
            for (int k = 0; k < 32; ++k) {
                volatile float t = w[k] / X;
                uint8_t c = ora_e2m1_encode(t);
                int64_t col = b * 32 + k;
                codes[o * (d / 2) + col / 2] |= (uint8_t)(c << (4 * (col % 2)));
            }
        }
    return 0;
}

static inline uint8_t fp4_at(const uint8_t* codes, int64_t d, int64_t o, int64_t k)
{
    return (uint8_t)((codes[o * (d / 2) + k / 2] >> (4 * (k % 2))) & 0xfu);
}

/* w_hat = fp16_RN(e2m1 * 2^(e - 127)): out [O][d] fp16 bits. */
int ora_dequant_mxfp4(const uint8_t* codes, const uint8_t* scales, int64_t O, int64_t d, uint16_t* out)
{
    if (O < 0 || d < 0 || d % 32 != 0) return -1;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t k = 0; k < d; ++k)
            out[o * d + k] = ora_f64_to_f16(ora_e2m1_decode(fp4_at(codes, d, o, k)) *
                                            ora_e8m0_decode(scales[o * (d / 32) + k / 32]));
    return 0;
}

/* codes [O][d/2], scales [O][d/16] E4M3, *tensor_scale fp32.  Returns 0 or -1. */
int ora_quantize_nvfp4(const float* W, int64_t O, int64_t d, uint8_t* codes, uint8_t* scales,
                       float* tensor_scale)
{
    if (O < 0 || d < 0 || d % 16 != 0) return -1;
    memset(codes, 0, (size_t)(O * (d / 2)));
    float amax_t = 0.0f;
    for (int64_t i = 0; i < O * d; ++i)
        if (fabsf(W[i]) > amax_t) amax_t = fabsf(W[i]);
    volatile float st = amax_t / (6.0f * 448.0f);
    if (!(st > 0.0f)) st = 1.0f;
    *tensor_scale = st;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t b = 0; b < d / 16; ++b) {
            const float* w = W + o * d + b * 16;
            float amax = 0.0f;
            for (int k = 0; k < 16; ++k)
                if (fabsf(w[k]) > amax) amax = fabsf(w[k]);
            volatile float six_st = 6.0f * st;
            volatile float sb = amax / six_st;
            uint8_t S = ora_e4m3_encode(sb);
            scales[o * (d / 16) + b] = S;
            volatile float dec = (float)ora_e4m3_decode(S);
            volatile float full = dec * st;
            for (int k = 0; k < 16; ++k) {
                uint8_t c = 0;
                if (full > 0.0f) {
                    volatile float t = w[k] / full;
                    c = ora_e2m1_encode(t);
                }
                int64_t col = b * 16 + k;
                codes[o * (d / 2) + col / 2] |= (uint8_t)(c << (4 * (col % 2)));
            }
        }
    return 0;
}

/* w_hat = fp16_RN(e2m1 * e4m3 * s_t), the product taken exactly: out [O][d] fp16 bits. */
int ora_dequant_nvfp4(const uint8_t* codes, const uint8_t* scales, float tensor_scale, int64_t O, int64_t d,
                      uint16_t* out)
{
    if (O < 0 || d < 0 || d % 16 != 0) return -1;
    for (int64_t o = 0; o < O; ++o)
        for (int64_t k = 0; k < d; ++k)
            out[o * d + k] = ora_f64_to_f16(ora_e2m1_decode(fp4_at(codes, d, o, k)) *
                                            ora_e4m3_decode(scales[o * (d / 16) + k / 16]) *
                                            (double)tensor_scale);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* FP8 activations for W4A8 (GlowQ pages: W4A8 alongside W4A16, Tables      */
/* 14-15 of the thelatestinai.com page; the format is not defined there).    */
/* ------------------------------------------------------------------------ */

/*
 * Readings: each token (row of X) gets one fp32 scale s = amax_row / 448
 * (1 for an all-zero row); codes = E4M3(x / s) rounded to nearest even and
 * saturating; the dequantised activation is the exact product dec(code) * s.
 * The whole layer (base product and the projection R) consumes the
 * dequantised activations.
 * X: T x d fp16 bits.  codes: T x d bytes, scales: T floats.
 */
int ora_quantize_act_e4m3(const uint16_t* X, int64_t T, int64_t d, uint8_t* codes, float* scales)
{
    if (T < 0 || d < 0) return -1;
    for (int64_t t = 0; t < T; ++t) {
        float amax = 0.0f;
        for (int64_t k = 0; k < d; ++k) {
            float a = fabsf((float)ora_f16_to_f64(X[t * d + k]));
            if (a > amax) amax = a;
        }
        volatile float s = amax / 448.0f;
        if (!(s > 0.0f)) s = 1.0f;
        scales[t] = s;
        for (int64_t k = 0; k < d; ++k) {
            volatile float q = (float)ora_f16_to_f64(X[t * d + k]) / s;
            codes[t * d + k] = ora_e4m3_encode(q);
        }
    }
    return 0;
}

/* out: T x d float64, dec(code) * s exactly. */
int ora_dequant_act_e4m3(const uint8_t* codes, const float* scales, int64_t T, int64_t d, double* out)
{
    if (T < 0 || d < 0) return -1;
    for (int64_t t = 0; t < T; ++t)
        for (int64_t k = 0; k < d; ++k)
            out[t * d + k] = ora_e4m3_decode(codes[t * d + k]) * (double)scales[t];
    return 0;
}
