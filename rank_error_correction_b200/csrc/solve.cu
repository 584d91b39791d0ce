// solve.cu -- the offline group solve on the GPU (GlowQ pages: papernotes.org
// summary, key designs 1-3; thelatestinai.com GlowQ page, Tables 11-12: exact
// vs randomised SVD of the covariance-aligned core, oversampling p and power
// iterations q).
//
// For one input-sharing group with stacked quantisation error
// E_cat = [E_1; ...; E_m] (E_i = W_i - w_hat_i) and input covariance root
// Sx^{1/2}, the shared factors minimise ||(E_cat - A B) Sx^{1/2}||_F at rank r:
//   E_w = E_cat Sx^{1/2}                    (whitened error, M x d)
//   Halko randomised SVD of E_w with test matrix Omega (d x l, l = r + p):
//     Y = E_w Omega, Q = orth(Y); q times: Q = orth(E_w orth(E_w^T Q))
//     Bs = Q^T E_w (l x d), Bs = U_b S V^T (eigen-decomposition of Bs Bs^T)
//   A = Q U_b,r S_r^{1/2},  B = S_r^{1/2} V_r^T Sx^{+1/2}
//   g_ec = sum_{j<=r} sigma_j^2 / ||E_w||_F^2   (GSVD energy capture)
// The pages take the thin QR core M = R_e Sx^{1/2} of E_cat first; E_w = Q_e M
// with Q_e orthonormal, so E_w and M share singular values and right vectors
// and every Halko iterate of E_w is Q_e times the iterate of M: the factors
// are the same, and working on E_w directly trades the QR of the tall E_cat
// for one more tall-skinny product per step.
// Arithmetic is float64 throughout (DMMA tensor cores for the products).
// orth() is CholeskyQR2: Q = Y R^{-1} with R from the Cholesky factor of Y^T Y,
// applied twice; a non-positive pivot records GLOWQ_ERR_NUMERIC.
#include <cmath>

#include "common.cuh"
#include "internal.cuh"

namespace glowq {

// ---------------------------------------------------------------------------
// Stacked error rows in float64: E[o][k] = W[o][k] - fp16((q - z) s) (exact).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) error_rows_f64_kernel(const float* __restrict__ W,
                                                              const uint32_t* __restrict__ q,
                                                              const __half* __restrict__ s,
                                                              const uint8_t* __restrict__ z, int64_t O, int64_t d,
                                                              double* __restrict__ E) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;   // one packed word
    if (i >= O * (d / 8)) return;
    const int64_t o = i / (d / 8), k0 = (i % (d / 8)) * 8;
    const int64_t g = o * (d / 128) + k0 / 128;
    const uint32_t w = q[qword_index(o, i % (d / 8), d)];
    const float sc = __half2float(s[g]);
    const int zz = z[g];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int c = (int)((w >> (4 * j)) & 0xfu);
        const float wh = __half2float(__float2half_rn((float)(c - zz) * sc));   // (q - z) s is exact in fp32
        E[o * d + k0 + j] = (double)W[o * d + k0 + j] - (double)wh;
    }
}

// ---------------------------------------------------------------------------
// C (M x N) = op(A) (M x K) op(B) (K x N), row-major with leading dimensions;
// op(A)[i][k] = TA ? A[k][i] : A[i][k], likewise B.  scale_cols: optional
// per-column factor of the result.  A CTA computes a 64 x 64 tile with four
// warps of 32 x 32, K in steps of 16 through shared memory, m8n8k4 DMMA.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void dmma_884(double c[2], double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                 : "+d"(c[0]), "+d"(c[1])
                 : "d"(a), "d"(b));
}

template <bool TA, bool TB>
__global__ void __launch_bounds__(128) dgemm_kernel(int M, int N, int K, const double* __restrict__ A, int64_t lda,
                                                     const double* __restrict__ B, int64_t ldb, double* __restrict__ C,
                                                     int64_t ldc, const double* __restrict__ scale_cols) {
    __shared__ double As[16][64 + 1];   // [k][m]
    __shared__ double Bs[16][64 + 1];   // [k][n]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = warp & 1, wn = warp >> 1;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    double acc[4][4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    for (int k0 = 0; k0 < K; k0 += 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int idx = tid + e * 128;   // 0 .. 1023
            int mi, kk;
            if (TA) { mi = idx & 63; kk = idx >> 6; }   // consecutive threads: consecutive m
            else { kk = idx & 15; mi = idx >> 4; }      // consecutive threads: consecutive k
            const int gm = m0 + mi, gk = k0 + kk;
            double v = 0.0;
            if (gm < M && gk < K) v = TA ? A[(int64_t)gk * lda + gm] : A[(int64_t)gm * lda + gk];
            As[kk][mi] = v;
            int ni, kb;
            if (TB) { kb = idx & 15; ni = idx >> 4; }
            else { ni = idx & 63; kb = idx >> 6; }
            const int gn = n0 + ni, gkb = k0 + kb;
            double u = 0.0;
            if (gn < N && gkb < K) u = TB ? B[(int64_t)gn * ldb + gkb] : B[(int64_t)gkb * ldb + gn];
            Bs[kb][ni] = u;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; kk += 4) {
            double af[4], bf[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) af[i] = As[kk + (lane & 3)][wm * 32 + i * 8 + (lane >> 2)];
#pragma unroll
            for (int j = 0; j < 4; ++j) bf[j] = Bs[kk + (lane & 3)][wn * 32 + j * 8 + (lane >> 2)];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) dmma_884(acc[i][j], af[i], bf[j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int gm = m0 + wm * 32 + i * 8 + (lane >> 2);
                const int gn = n0 + wn * 32 + j * 8 + 2 * (lane & 3) + h;
                if (gm < M && gn < N) {
                    double v = acc[i][j][h];
                    if (scale_cols) v *= scale_cols[gn];
                    C[(int64_t)gm * ldc + gn] = v;
                }
            }
}

static cudaError_t dgemm(bool ta, bool tb, int M, int N, int K, const double* A, int64_t lda, const double* B,
                         int64_t ldb, double* C, int64_t ldc, cudaStream_t st, const double* scale_cols = nullptr) {
    const dim3 grid((N + 63) / 64, (M + 63) / 64);
    if (!ta && !tb) dgemm_kernel<false, false><<<grid, 128, 0, st>>>(M, N, K, A, lda, B, ldb, C, ldc, scale_cols);
    else if (ta && !tb) dgemm_kernel<true, false><<<grid, 128, 0, st>>>(M, N, K, A, lda, B, ldb, C, ldc, scale_cols);
    else if (!ta && tb) dgemm_kernel<false, true><<<grid, 128, 0, st>>>(M, N, K, A, lda, B, ldb, C, ldc, scale_cols);
    else dgemm_kernel<true, true><<<grid, 128, 0, st>>>(M, N, K, A, lda, B, ldb, C, ldc, scale_cols);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// One CTA: R^{-1} of the upper Cholesky factor of the SPD l x l matrix G
// (G = R^T R).  Writes Rinv (upper triangular, l x l).  A non-positive pivot
// records GLOWQ_ERR_NUMERIC in *err and leaves Rinv zero.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) chol_inv_kernel(const double* __restrict__ G, int l, double* __restrict__ Rinv,
                                                       unsigned int* err) {
    extern __shared__ double sm[];
    double* R = sm;              // [l][l], the factor in place of G
    double* X = sm + l * l;      // [l][l], the inverse
    __shared__ int bad;
    const int tid = threadIdx.x, nt = blockDim.x;
    if (tid == 0) bad = 0;
    for (int i = tid; i < l * l; i += nt) {
        R[i] = G[i];
        X[i] = 0.0;
    }
    __syncthreads();
    for (int j = 0; j < l; ++j) {
        if (tid == 0) {
            const double pv = R[j * l + j];
            if (!(pv > 0.0)) bad = 1;
            R[j * l + j] = pv > 0.0 ? sqrt(pv) : 1.0;
        }
        __syncthreads();
        const double rjj = R[j * l + j];
        for (int c = j + 1 + tid; c < l; c += nt) R[j * l + c] /= rjj;
        __syncthreads();
        for (int i = tid; i < (l - j - 1) * (l - j - 1); i += nt) {   // trailing update
            const int a = j + 1 + i / (l - j - 1), b = j + 1 + i % (l - j - 1);
            if (b >= a) R[a * l + b] -= R[j * l + a] * R[j * l + b];
        }
        __syncthreads();
    }
    // inverse of the upper factor, column by column (back substitution)
    for (int c = tid; c < l; c += nt) {
        for (int i = c; i >= 0; --i) {
            double v = (i == c) ? 1.0 : 0.0;
            for (int k = i + 1; k <= c; ++k) v -= R[i * l + k] * X[k * l + c];
            X[i * l + c] = v / R[i * l + i];
        }
    }
    __syncthreads();
    for (int i = tid; i < l * l; i += nt) Rinv[i] = bad ? 0.0 : X[i];
    if (tid == 0 && bad && err) atomicCAS(err, 0u, (unsigned int)GLOWQ_ERR_NUMERIC);
}

// ---------------------------------------------------------------------------
// One CTA: eigen-decomposition of the symmetric l x l matrix S (l even,
// l <= 112) by parallel cyclic Jacobi rotations (round-robin pairing, each
// round rotates l/2 disjoint pairs).  Outputs the eigenvalues in descending
// order and the matching eigenvectors as columns of U (l x l).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) jacobi_eig_kernel(const double* __restrict__ S_in, int l, int sweeps,
                                                         double* __restrict__ lam, double* __restrict__ U) {
    extern __shared__ double sm[];
    double* S = sm;                    // [l][l]
    double* V = sm + l * l;            // [l][l]
    double* cs = V + l * l;            // [l/2][2] rotation (c, s) of each pair
    int* pp = reinterpret_cast<int*>(cs + l);   // [l/2][2] pair members
    int* perm = pp + l;                // [l] round-robin order
    const int tid = threadIdx.x, nt = blockDim.x, h = l / 2;
    for (int i = tid; i < l * l; i += nt) {
        S[i] = S_in[i];
        V[i] = ((i / l) == (i % l)) ? 1.0 : 0.0;
    }
    for (int i = tid; i < l; i += nt) perm[i] = i;
    __syncthreads();
    for (int sw = 0; sw < sweeps; ++sw) {
        for (int rd = 0; rd < l - 1; ++rd) {
            for (int k = tid; k < h; k += nt) {
                int p = perm[k], q = perm[l - 1 - k];
                if (p > q) { const int t = p; p = q; q = t; }
                pp[2 * k] = p;
                pp[2 * k + 1] = q;
                const double apq = S[p * l + q];
                double c = 1.0, s = 0.0;
                if (apq != 0.0) {
                    const double tau = (S[q * l + q] - S[p * l + p]) / (2.0 * apq);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    s = t * c;
                }
                cs[2 * k] = c;
                cs[2 * k + 1] = s;
            }
            __syncthreads();
            for (int i = tid; i < h * l; i += nt) {   // columns p, q of S and V: S <- S J, V <- V J
                const int k = i / l, row = i % l;
                const int p = pp[2 * k], q = pp[2 * k + 1];
                const double c = cs[2 * k], s = cs[2 * k + 1];
                const double sp = S[row * l + p], sq = S[row * l + q];
                S[row * l + p] = c * sp - s * sq;
                S[row * l + q] = s * sp + c * sq;
                const double vp = V[row * l + p], vq = V[row * l + q];
                V[row * l + p] = c * vp - s * vq;
                V[row * l + q] = s * vp + c * vq;
            }
            __syncthreads();
            for (int i = tid; i < h * l; i += nt) {   // rows p, q of S: S <- J^T S
                const int k = i / l, col = i % l;
                const int p = pp[2 * k], q = pp[2 * k + 1];
                const double c = cs[2 * k], s = cs[2 * k + 1];
                const double sp = S[p * l + col], sq = S[q * l + col];
                S[p * l + col] = c * sp - s * sq;
                S[q * l + col] = s * sp + c * sq;
            }
            __syncthreads();
            if (tid == 0) {   // circle method: keep perm[0], rotate the rest by one
                const int last = perm[l - 1];
                for (int i = l - 1; i > 1; --i) perm[i] = perm[i - 1];
                perm[1] = last;
            }
            __syncthreads();
        }
    }
    if (tid == 0) {   // descending order of the eigenvalues (diagonal of S)
        for (int i = 0; i < l; ++i) perm[i] = i;
        for (int i = 1; i < l; ++i) {
            const int v = perm[i];
            int j = i - 1;
            while (j >= 0 && S[perm[j] * l + perm[j]] < S[v * l + v]) {
                perm[j + 1] = perm[j];
                --j;
            }
            perm[j + 1] = v;
        }
    }
    __syncthreads();
    for (int i = tid; i < l; i += nt) lam[i] = S[perm[i] * l + perm[i]];
    for (int i = tid; i < l * l; i += nt) U[i] = V[(i / l) * l + perm[i % l]];
}

// sum of squares of n doubles into *out (fp64 atomics; used for ||E_w||_F^2)
__global__ void __launch_bounds__(256) sumsq_kernel(const double* __restrict__ x, int64_t n, double* out) {
    double v = 0.0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        v += x[i] * x[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) atomicAdd(out, v);
}

// sigma_j = sqrt(max(lambda_j, 0)); per-column factors sqrt(sigma) and
// 1/sqrt(sigma) (0 for sigma = 0), and g_ec
__global__ void solve_scalars_kernel(const double* __restrict__ lam, int r, const double* __restrict__ ew2,
                                     double* __restrict__ sing, double* __restrict__ sq, double* __restrict__ inv,
                                     double* __restrict__ gec) {
    if (threadIdx.x != 0) return;
    double cap = 0.0;
    for (int j = 0; j < r; ++j) {
        const double sg = sqrt(lam[j] > 0.0 ? lam[j] : 0.0);
        sing[j] = sg;
        sq[j] = sqrt(sg);
        inv[j] = sg > 0.0 ? 1.0 / sqrt(sg) : 0.0;
        cap += sg * sg;
    }
    if (gec) *gec = (*ew2 > 0.0) ? cap / *ew2 : 1.0;
}

__global__ void __launch_bounds__(256) f64_to_f16_kernel(const double* __restrict__ x, int64_t n,
                                                          __half* __restrict__ y) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) y[i] = __double2half(x[i]);
}

// ---------------------------------------------------------------------------
// Host driver
// ---------------------------------------------------------------------------
static size_t al256(size_t x) { return (x + 255) / 256 * 256; }

size_t solve_workspace_bytes(int64_t M, int64_t d, int l) {
    return al256((size_t)M * d * 8) * 2 +       // E, E_w
           al256((size_t)M * l * 8) * 2 +       // Y, Q
           al256((size_t)d * l * 8) * 2 +       // Z, Zq
           al256((size_t)l * d * 8) +           // Bs
           al256((size_t)l * l * 8) * 3 +       // Gram, Rinv, U_b
           al256((size_t)l * 8) * 4 +           // lambda, sqrt sigma, 1/sqrt sigma, sigma
           256;                                 // ||E_w||^2
}

glowq_status group_solve_impl(const SolveModule* mods, int m, int64_t d, const double* Sh, const double* Shp,
                              int r, int p, int qit, const double* Omega, double* A, double* Bout, double* sing,
                              double* gec, uint16_t* A16, uint16_t* B16, void* workspace, unsigned int* err,
                              cudaStream_t st) {
    int64_t M = 0;
    for (int i = 0; i < m; ++i) M += mods[i].O;
    const int l = r + p;
    char* w = static_cast<char*>(workspace);
    auto take = [&](size_t bytes) { char* q = w; w += al256(bytes); return reinterpret_cast<double*>(q); };
    double* E = take((size_t)M * d * 8);
    double* Ew = take((size_t)M * d * 8);
    double* Y = take((size_t)M * l * 8);
    double* Q = take((size_t)M * l * 8);
    double* Z = take((size_t)d * l * 8);
    double* Zq = take((size_t)d * l * 8);
    double* Bs = take((size_t)l * d * 8);
    double* G = take((size_t)l * l * 8);
    double* Rinv = take((size_t)l * l * 8);
    double* Ub = take((size_t)l * l * 8);
    double* lam = take((size_t)l * 8);
    double* sqs = take((size_t)l * 8);
    double* inv = take((size_t)l * 8);
    double* sing_ws = take((size_t)l * 8);
    double* ew2 = take(8);
    if (!sing) sing = sing_ws;
    cudaError_t e = cudaSuccess;
    // E_cat and E_w = E_cat Sx^{1/2}
    int64_t row = 0;
    for (int i = 0; i < m && e == cudaSuccess; ++i) {
        const int64_t words = mods[i].O * (d / 8);
        error_rows_f64_kernel<<<(unsigned)((words + 255) / 256), 256, 0, st>>>(
            mods[i].W, mods[i].q, reinterpret_cast<const __half*>(mods[i].s), mods[i].z, mods[i].O, d, E + row * d);
        e = cudaGetLastError();
        row += mods[i].O;
    }
    if (e == cudaSuccess) e = dgemm(false, false, (int)M, (int)d, (int)d, E, d, Sh, d, Ew, d, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(ew2, 0, 8, st);
    if (e == cudaSuccess) {
        sumsq_kernel<<<1024, 256, 0, st>>>(Ew, M * d, ew2);
        e = cudaGetLastError();
    }
    const size_t chol_smem = (size_t)2 * l * l * 8;
    const size_t jac_smem = (size_t)2 * l * l * 8 + (size_t)l * 8 + (size_t)3 * l * 4;
    static bool opted = false;
    if (e == cudaSuccess && !opted) {
        e = cudaFuncSetAttribute(chol_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 2 * 112 * 112 * 8);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     2 * 112 * 112 * 8 + 112 * 8 + 3 * 112 * 4);
        opted = e == cudaSuccess;
    }
    // orth(X, rows): X <- X R^{-1} twice (CholeskyQR2), through `tmp`
    auto orth = [&](double* X, double* tmp, int rows) -> cudaError_t {
        for (int pass = 0; pass < 2; ++pass) {
            cudaError_t ee = dgemm(true, false, l, l, rows, X, l, X, l, G, l, st);   // G = X^T X
            if (ee != cudaSuccess) return ee;
            chol_inv_kernel<<<1, 256, chol_smem, st>>>(G, l, Rinv, err);
            if ((ee = cudaGetLastError()) != cudaSuccess) return ee;
            ee = dgemm(false, false, rows, l, l, X, l, Rinv, l, tmp, l, st);          // tmp = X R^{-1}
            if (ee != cudaSuccess) return ee;
            ee = cudaMemcpyAsync(X, tmp, (size_t)rows * l * 8, cudaMemcpyDeviceToDevice, st);
            if (ee != cudaSuccess) return ee;
        }
        return cudaSuccess;
    };
    // range finder with q power iterations
    if (e == cudaSuccess) e = dgemm(false, false, (int)M, l, (int)d, Ew, d, Omega, l, Q, l, st);   // Y = E_w Omega
    if (e == cudaSuccess) e = orth(Q, Y, (int)M);
    for (int it = 0; it < qit && e == cudaSuccess; ++it) {
        e = dgemm(true, false, (int)d, l, (int)M, Ew, d, Q, l, Z, l, st);                        // Z = E_w^T Q
        if (e == cudaSuccess) e = orth(Z, Zq, (int)d);
        if (e == cudaSuccess) e = dgemm(false, false, (int)M, l, (int)d, Ew, d, Z, l, Q, l, st); // Y = E_w Z
        if (e == cudaSuccess) e = orth(Q, Y, (int)M);
    }
    // small SVD: Bs = Q^T E_w (l x d), Bs Bs^T = U_b diag(lambda) U_b^T
    if (e == cudaSuccess) e = dgemm(true, false, l, (int)d, (int)M, Q, l, Ew, d, Bs, d, st);
    if (e == cudaSuccess) e = dgemm(false, true, l, l, (int)d, Bs, d, Bs, d, G, l, st);
    if (e == cudaSuccess) {
        jacobi_eig_kernel<<<1, 256, jac_smem, st>>>(G, l, 16, lam, Ub);
        e = cudaGetLastError();
    }
    if (e == cudaSuccess) {
        solve_scalars_kernel<<<1, 32, 0, st>>>(lam, r, ew2, sing, sqs, inv, gec);
        e = cudaGetLastError();
    }
    // V_r S_r^{1/2} = Bs^T U_b,r S_r^{-1/2} (d x r, into Z)
    if (e == cudaSuccess) e = dgemm(true, false, (int)d, r, l, Bs, d, Ub, l, Z, r, st, inv);
    // A = Q U_b,r S_r^{1/2} (M x r)
    if (e == cudaSuccess) e = dgemm(false, false, (int)M, r, l, Q, l, Ub, l, A, r, st, sqs);
    // B = S_r^{1/2} V_r^T Sx^{+1/2}: (V_r S_r^{1/2})^T (r x d) times Shp
    if (e == cudaSuccess) e = dgemm(true, false, r, (int)d, (int)d, Z, r, Shp, d, Bout, d, st);
    if (e == cudaSuccess && A16) {
        f64_to_f16_kernel<<<(unsigned)((M * r + 255) / 256), 256, 0, st>>>(A, M * r, reinterpret_cast<__half*>(A16));
        e = cudaGetLastError();
    }
    if (e == cudaSuccess && B16) {
        f64_to_f16_kernel<<<(unsigned)(((int64_t)r * d + 255) / 256), 256, 0, st>>>(Bout, (int64_t)r * d,
                                                                                     reinterpret_cast<__half*>(B16));
        e = cudaGetLastError();
    }
    return e == cudaSuccess ? GLOWQ_OK : GLOWQ_ERR_CUDA;
}

}  // namespace glowq
