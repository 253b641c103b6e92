// Factorization of the damped Hessian: U upper with (H + lambda I)^-1 = U^T U.
//
// GPTQ-2D (two-sided adaptive rounding), sections 2 and 4: the feedback of adaptive
// rounding is a triangular factor of the inverse Gram matrix, and the factorization costs
// O(n^3). Route taken here (the cheapest exact one, 2/3 n^3 flops):
//   A = H + lambda I = Ubar Ubar^T     Ubar upper: Cholesky run from the last column back
//   U = Ubar^-1                        upper triangular inverse
// Then U^T U = Ubar^-T Ubar^-1 = A^-1, and since the upper factor of A^-1 with a positive
// diagonal is unique, this is the U of the chol -> inverse -> chol route.
//
// Recursive, bottom-right half first (factor_rec below): the work is four large GEMMs per
// split (tensor cores through gemm_f32) and one-CTA register-tiled kernels on the
// 128-column diagonal leaves (diag_ul_inv_kernel).
#pragma once

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"

namespace gptq {

constexpr int FACTOR_NB = 128;

// One CTA: UL-Cholesky of an nb x nb symmetric block (upper triangle read) and the inverse of
// its factor. On exit U's block holds U_pp = Ubar_pp^-1 (upper; strictly lower part zeroed),
// where A_pp = Ubar_pp Ubar_pp^T; Ubar_pp itself is used by no later step and is not stored.
//
// Register-tiled sweep: thread (ty, tx) of a 16 x 16 grid holds the 8 x 8 entries with rows
// ty + 16 a and columns tx + 16 b of one matrix M. Before step c, M's columns <= c hold the
// leading block still to be factored and its columns > c hold, for rows < c, the partial sums
// P[i][j] = sum_{k > c} Ubar[i][k] X[k][j] of the inverse X = Ubar^-1 (rows > c of M already
// are rows of X). Step c (from the last column to the first), with one barrier:
//   column c (rows <= c) and row c (columns > c) of M are published to shared memory;
//   pivot d = M[c][c], u_i = M[i][c] / sqrt(d) (Ubar's column c), row c of X is
//   x_c = 1/sqrt(d), x_j = -P[c][j] / sqrt(d);
//   rows i < c get M[i][j] += u_i v_j with v_j = -u_j (j < c: the Cholesky update),
//   v_c = x_c (column c restarts as a partial sum), v_j = x_j (j > c: the inverse update).
// A pivot <= 0 (or NaN) records GPTQ_ERR_NOT_PD with info = col_base + c and continues with a
// unit pivot so that the kernel always finishes.
constexpr int DIAG_THREADS = 256;

template <typename T>
__global__ __launch_bounds__(DIAG_THREADS) void diag_ul_inv_kernel(const T *A, long long lda,
                                                                   T *U, long long ldu, int nb,
                                                                   long long col_base) {
    // wb[c' ] = M[c'][c] for c' < c (column c), -1 at c, M[c][c'] for c' > c (row c); the
    // pivot M[c][c] separately. Then u_i = ipiv wb[i] (i < c) and v_j = -ipiv wb[j].
    __shared__ T wb[2][FACTOR_NB];
    __shared__ T dpiv[2];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    T M[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int i = ty + 16 * a, j = tx + 16 * b;
            T v = T(0);
            if (i < nb && j < nb) v = j >= i ? A[(long long)i * lda + j] : A[(long long)j * lda + i];
            M[a][b] = v;
        }
    int buf = 0;
#pragma unroll
    for (int b = 7; b >= 0; --b) {
        for (int cc = 15; cc >= 0; --cc) {
            const int c = 16 * b + cc;
            if (c >= nb) continue;
            if (tx == cc) {
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const int i = ty + 16 * a;
                    if (i < c) wb[buf][i] = M[a][b];
                    else if (i == c) { wb[buf][c] = T(-1); dpiv[buf] = M[a][b]; }
                }
            }
            if (ty == cc) {
#pragma unroll
                for (int b2 = 0; b2 < 8; ++b2) {
                    const int j = tx + 16 * b2;
                    if (j > c && j < nb) wb[buf][j] = M[b][b2];
                }
            }
            __syncthreads();
            const T d = dpiv[buf];
            const bool bad = !(d > T(0)) || !isfinite((double)d);
            if (bad && tid == 0) report(GPTQ_ERR_NOT_PD, col_base + c);
            // 1/sqrt(d): hardware estimate refined by one Newton step
            const T dd = bad ? T(1) : d;
            T ipiv = rsqrt(dd);
            ipiv = ipiv * (T(1.5) - T(0.5) * dd * ipiv * ipiv);
            T u[8], v[8];
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                const int i = ty + 16 * a;
                u[a] = i < c ? wb[buf][i] * ipiv : T(0);
            }
#pragma unroll
            for (int b2 = 0; b2 < 8; ++b2) {
                const int j = tx + 16 * b2;
                v[b2] = j < nb ? -ipiv * wb[buf][j] : T(0);
            }
            if (tx == cc) {
#pragma unroll
                for (int a = 0; a < 8; ++a)
                    if (ty + 16 * a < c) M[a][b] = T(0);
            }
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                if (ty + 16 * a < c) {
#pragma unroll
                    for (int b2 = 0; b2 < 8; ++b2) M[a][b2] = fma(u[a], v[b2], M[a][b2]);
                }
            }
            if (ty == cc) {
#pragma unroll
                for (int b2 = 0; b2 < 8; ++b2) {
                    const int j = tx + 16 * b2;
                    if (j >= c && j < nb) M[b][b2] = v[b2];
                }
            }
            buf ^= 1;
        }
    }
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            const int i = ty + 16 * a, j = tx + 16 * b;
            if (i < nb && j < nb) U[(long long)i * ldu + j] = j >= i ? M[a][b] : T(0);
        }
}

// U_pp = inverse of the UL factor of the nb x nb block at A (nb <= FACTOR_NB).
template <typename T>
inline int diag_ul_inv(const T *A, long long lda, T *U, long long ldu, int nb, long long col_base,
                       cudaStream_t s) {
    diag_ul_inv_kernel<T><<<1, DIAG_THREADS, 0, s>>>(A, lda, U, ldu, nb, col_base);
    return launch_status();
}

// A_work = H + lambda I (full copy), lambda = lambda_rel * mean(diag H) written to *lam.
__global__ void damp_mean_kernel(const float *H, long long ldh, int n, float lambda_rel,
                                 float *lam) {
    __shared__ double part[32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float d = H[(long long)i * ldh + i];
        if (!isfinite(d)) report(GPTQ_ERR_NONFINITE, (long long)i * ldh + i);
        acc += d;
    }
    acc = warp_sum_d(acc);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
        v = warp_sum_d(v);
        if (threadIdx.x == 0) *lam = (float)((double)lambda_rel * v / (double)n);
    }
}

__global__ void copy_damped_kernel(const float *H, long long ldh, float *A, long long lda,
                                   int n, const float *lam) {
    const float l = *lam;
    const long long total = (long long)n * n;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(idx / n), j = (int)(idx % n);
        float v = H[(long long)i * ldh + j];
        if (i == j) v += l;
        A[(long long)i * lda + j] = v;
    }
}

// Recursive UL factorization + inverse of the diagonal block [r0, r1) of A (upper triangle
// read): A_blk = Ubar Ubar^T, and U[r0:r1, r0:r1] = Ubar^-1 is written. With the block split
// at m (a multiple of FACTOR_NB) into 1 = [r0, m) and 2 = [m, r1):
//   U22            <- recursion on block 2 (bottom-right first)
//   Ubar12 = A12 U22^T             (kept transposed, S12 = U22 A12^T, in A's lower-left block)
//   A11   -= Ubar12 Ubar12^T       (upper triangle)
//   U11            <- recursion on block 1
//   U12 = -U11 (Ubar12 U22)        (the product Ubar12 U22 is staged in A12's place)
// This is the block form of Ubar U = I. Every step is a large GEMM except the 128-wide leaves
// (one-CTA diagonal kernel); A's strictly lower triangle is used as scratch, so nothing beyond
// the n x n work matrix is needed.
inline int factor_rec(float *A, long long lda, float *U, long long ldu, int r0, int r1,
                      cudaStream_t s) {
    const int len = r1 - r0;
    if (len <= FACTOR_NB)
        return diag_ul_inv<float>(A + (long long)r0 * lda + r0, lda, U + (long long)r0 * ldu + r0,
                                  ldu, len, r0, s);
    const int m = r0 + (ceil_div(len, FACTOR_NB) / 2) * FACTOR_NB;
    const int n1 = m - r0, n2 = r1 - m;
    if (int st = factor_rec(A, lda, U, ldu, m, r1, s)) return st;
    float *A12 = A + (long long)r0 * lda + m;        // n1 x n2
    float *S12 = A + (long long)m * lda + r0;        // n2 x n1 scratch (below the diagonal)
    const float *U22 = U + (long long)m * ldu + m;   // n2 x n2 upper
    // S12 = U22 A12^T
    auto p2 = gemm_args<float, float>(n2, n1, n2, U22, ldu, 0, A12, lda, 1, S12, lda, 1.f, 0.f);
    p2.a_upper = 1;
    if (int st = gemm_f32(p2, s)) return st;
    // A11 -= S12^T S12 (upper)
    auto p3 = gemm_args<float, float>(n1, n1, n2, S12, lda, 1, S12, lda, 0,
                                      A + (long long)r0 * lda + r0, lda, -1.f, 1.f);
    p3.c_upper = 1;
    if (int st = gemm_f32(p3, s)) return st;
    if (int st = factor_rec(A, lda, U, ldu, r0, m, s)) return st;
    // A12 <- T1 = Ubar12 U22 = S12^T U22
    auto p5 = gemm_args<float, float>(n1, n2, n2, S12, lda, 1, U22, ldu, 0, A12, lda, 1.f, 0.f);
    p5.b_upper = 1;
    if (int st = gemm_f32(p5, s)) return st;
    // U12 = -U11 T1
    auto p6 = gemm_args<float, float>(n1, n2, n1, U + (long long)r0 * ldu + r0, ldu, 0, A12, lda, 0,
                                      U + (long long)r0 * ldu + m, ldu, -1.f, 0.f);
    p6.a_upper = 1;
    return gemm_f32(p6, s);
}

// A (n x n, lda) holds the damped matrix on entry (upper triangle read; the rest of A is
// scratch); U (n x n, ldu) receives the inverse factor (upper; its strictly lower part must
// be zero on entry and stays zero).
inline int factor_ul_inverse(float *A, long long lda, float *U, long long ldu, int n,
                             float * /*unused*/, cudaStream_t s) {
    return factor_rec(A, lda, U, ldu, 0, n, s);
}

}  // namespace gptq
