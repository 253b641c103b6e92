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
// Blocked, bottom-right first, with blocks of NB columns. For block p (rows r0..r1):
//   1. diag:  A_pp = Ubar_pp Ubar_pp^T  and  U_pp = Ubar_pp^-1          (one CTA)
//      (Ubar_pp itself is used by no later step)
//   2. panel: Ubar[0:r0, p] = A[0:r0, p] U_pp^T                           (GEMM)
//   3. syrk:  A[0:r0, 0:r0] -= Ubar[0:r0, p] Ubar[0:r0, p]^T (upper)       (GEMM)
//   4. row p of U:  U[p, r1:] = -U_pp (Ubar[p, r1:] U[r1:, r1:])          (two GEMMs)
// Step 4 uses Ubar's row block p (finished by earlier, later-indexed blocks) and the
// already finished trailing part of U.
#pragma once

#include "common.cuh"
#include "gemm_simt.cuh"

namespace gptq {

constexpr int FACTOR_NB = 128;

// One CTA: UL-Cholesky of an nb x nb symmetric block (upper triangle read) followed by the
// inverse of its factor, in place in shared memory. On exit U's block holds
// U_pp = Ubar_pp^-1 (upper; strictly lower part zeroed), where A_pp = Ubar_pp Ubar_pp^T.
// Ubar_pp itself is not needed by any later step and is not stored.
// Column c is processed from the last to the first: pivot, scaled column above it, update
// of the leading block; then row c of the inverse, which only needs Ubar's row c (saved
// first) and the rows of the inverse below it (already in place).
// A pivot <= 0 (or NaN) records GPTQ_ERR_NOT_PD with info = col_base + c and continues with a
// unit pivot so that the kernel always finishes.
template <typename T>
__global__ __launch_bounds__(512) void diag_ul_inv_kernel(const T *A, long long lda, T *U,
                                                          long long ldu, int nb,
                                                          long long col_base) {
    extern __shared__ __align__(16) unsigned char smraw[];
    T *S = reinterpret_cast<T *>(smraw);
    T *rowc = S + nb * (nb + 1);
    const int LD = nb + 1;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    for (int idx = tid; idx < nb * nb; idx += blockDim.x) {
        const int i = idx / nb, j = idx % nb;
        S[i * LD + j] = (j >= i) ? A[(long long)i * lda + j] : T(0);
    }
    __syncthreads();
    for (int c = nb - 1; c >= 0; --c) {
        const T d = S[c * LD + c];
        const bool bad = !(d > T(0)) || !isfinite((double)d);
        if (bad && tid == 0) report(GPTQ_ERR_NOT_PD, col_base + c);
        const T piv = bad ? T(1) : sqrt(d);
        __syncthreads();
        for (int i = tid; i < c; i += blockDim.x) S[i * LD + c] = S[i * LD + c] / piv;
        for (int k = c + 1 + tid; k < nb; k += blockDim.x) rowc[k] = S[c * LD + k];
        __syncthreads();
        for (int i = warp; i < c; i += nw) {
            const T sic = S[i * LD + c];
            for (int j = i + lane; j < c; j += 32) S[i * LD + j] -= sic * S[j * LD + c];
        }
        const T xcc = T(1) / piv;
        for (int j = c + 1 + warp; j < nb; j += nw) {
            T acc = T(0);
            for (int k = c + 1 + lane; k <= j; k += 32) acc += rowc[k] * S[k * LD + j];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) S[c * LD + j] = -xcc * acc;
        }
        if (tid == 0) S[c * LD + c] = xcc;
        __syncthreads();
    }
    for (int idx = tid; idx < nb * nb; idx += blockDim.x) {
        const int i = idx / nb, j = idx % nb;
        U[(long long)i * ldu + j] = (j >= i) ? S[i * LD + j] : T(0);
    }
}

template <typename T>
inline size_t diag_smem(int nb) { return ((size_t)nb * (nb + 1) + nb) * sizeof(T); }

// U_pp = inverse of the UL factor of the nb x nb block at A (nb <= FACTOR_NB).
template <typename T>
inline int diag_ul_inv(const T *A, long long lda, T *U, long long ldu, int nb, long long col_base,
                       cudaStream_t s) {
    const size_t smem = diag_smem<T>(FACTOR_NB);
    cudaFuncSetAttribute(diag_ul_inv_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    diag_ul_inv_kernel<T><<<1, 512, diag_smem<T>(nb), s>>>(A, lda, U, ldu, nb, col_base);
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

// Blocked UL factorization + inverse. A (n x n, lda) holds the damped matrix on entry (upper
// triangle read) and Ubar on exit (upper triangle); U (n x n, ldu) receives the inverse
// factor (upper; strictly lower part zero). T is scratch of FACTOR_NB x n floats.
inline int factor_ul_inverse(float *A, long long lda, float *U, long long ldu, int n,
                             float *T, cudaStream_t s) {
    const int P = ceil_div(n, FACTOR_NB);
    for (int p = P - 1; p >= 0; --p) {
        const int r0 = p * FACTOR_NB;
        const int r1 = min(n, r0 + FACTOR_NB);
        const int nb = r1 - r0;
        if (int st = diag_ul_inv<float>(A + (long long)r0 * lda + r0, lda,
                                        U + (long long)r0 * ldu + r0, ldu, nb, r0, s))
            return st;
        if (r0 > 0) {
            // 2. panel: A[0:r0, r0:r1] = A[0:r0, r0:r1] * U_pp^T  (in place: one column tile)
            auto pa = gemm_args<float, float>(r0, nb, nb, A + r0, lda, 0,
                                              U + (long long)r0 * ldu + r0, ldu, 1, A + r0, lda,
                                              1.f, 0.f);
            if (int st = gemm_simt(pa, s)) return st;
            // 3. syrk: A[0:r0, 0:r0] -= P P^T (upper)
            auto ps = gemm_args<float, float>(r0, r0, nb, A + r0, lda, 0, A + r0, lda, 1, A, lda,
                                              -1.f, 1.f);
            ps.c_upper = 1;
            if (int st = gemm_simt(ps, s)) return st;
        }
        if (r1 < n) {
            const int w = n - r1;
            // 4a. T = Ubar[r0:r1, r1:n] * U[r1:n, r1:n]   (U upper)
            auto pt = gemm_args<float, float>(nb, w, w, A + (long long)r0 * lda + r1, lda, 0,
                                              U + (long long)r1 * ldu + r1, ldu, 0, T, n, 1.f, 0.f);
            pt.b_upper = 1;
            if (int st = gemm_simt(pt, s)) return st;
            // 4b. U[r0:r1, r1:n] = -U_pp * T   (U_pp upper)
            auto pu = gemm_args<float, float>(nb, w, nb, U + (long long)r0 * ldu + r0, ldu, 0, T, n,
                                              0, U + (long long)r0 * ldu + r1, ldu, -1.f, 0.f);
            pu.a_upper = 1;
            if (int st = gemm_simt(pu, s)) return st;
        }
    }
    return GPTQ_OK;
}

}  // namespace gptq
