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
// Blocked and right-looking, last block first (factor_ul_inverse below): a chain of
// one-CTA leaf kernels and small panel GEMMs on a high-priority stream, with the trailing
// updates and the rows of the inverse as tensor-core GEMMs on two more streams.
#pragma once

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"

namespace gptq {

constexpr int FACTOR_NB = 128;

// One CTA: UL-Cholesky of an nb x nb symmetric block (upper triangle read) and the inverse of
// its factor. On exit U's block holds U_pp = Ubar_pp^-1 (upper; strictly lower part zeroed),
// where A_pp = Ubar_pp Ubar_pp^T; Ubar_pp itself is used by no later step and is not stored.
//
// Register-tiled sweep: thread (ty, tx) of a TG x TG grid holds the TS x TS entries with rows
// ty + TG a and columns tx + TG b of one matrix M (TG TS = 128). Before step c, M's columns <= c
// hold the leading block still to be factored and its columns > c hold, for rows < c, the
// partial sums P[i][j] = sum_{k > c} Ubar[i][k] X[k][j] of the inverse X = Ubar^-1 (rows > c of
// M already are rows of X). Step c (from the last column to the first), with one barrier:
//   column c (rows <= c) and row c (columns > c) of M are published to shared memory;
//   pivot d = M[c][c], u_i = M[i][c] / sqrt(d) (Ubar's column c), row c of X is
//   x_c = 1/sqrt(d), x_j = -P[c][j] / sqrt(d);
//   rows i < c get M[i][j] += u_i v_j with v_j = -u_j (j < c: the Cholesky update),
//   v_c = x_c (column c restarts as a partial sum), v_j = x_j (j > c: the inverse update).
// A pivot <= 0 (or NaN) records GPTQ_ERR_NOT_PD with info = col_base + c and continues with a
// unit pivot so that the kernel always finishes. fp32 blocks use 16 x 16 threads, fp64 blocks
// (the small Gram and extra-block factors of the intrinsic-LoRA step) 32 x 32, which shortens
// each step's dependent chain of fp64 FMAs.
template <typename T> struct DiagCfg { static constexpr int TG = 16, TS = 8; };
template <> struct DiagCfg<double> { static constexpr int TG = 32, TS = 4; };

template <typename T>
__global__ __launch_bounds__(DiagCfg<T>::TG * DiagCfg<T>::TG) void diag_ul_inv_kernel(
    const T *A, long long lda, T *U, long long ldu, int nb, long long col_base, const int *skip) {
    constexpr int TG = DiagCfg<T>::TG, TS = DiagCfg<T>::TS;
    pdl_wait_prev();
    pdl_launch_next();
    if (skip && *skip) return;
    // wb[c'] = M[c'][c] for c' < c (column c), -1 at c, M[c][c'] for c' > c (row c); the
    // pivot M[c][c] separately. Then u_i = ipiv wb[i] (i < c) and v_j = -ipiv wb[j].
    __shared__ T wb[2][FACTOR_NB];
    __shared__ T dpiv[2];
    const int tid = threadIdx.x, tx = tid % TG, ty = tid / TG;
    T M[TS][TS];
#pragma unroll
    for (int a = 0; a < TS; ++a)
#pragma unroll
        for (int b = 0; b < TS; ++b) {
            const int i = ty + TG * a, j = tx + TG * b;
            T v = T(0);
            if (i < nb && j < nb) v = j >= i ? A[(long long)i * lda + j] : A[(long long)j * lda + i];
            M[a][b] = v;
        }
    int buf = 0;
#pragma unroll
    for (int b = TS - 1; b >= 0; --b) {
        for (int cc = TG - 1; cc >= 0; --cc) {
            const int c = TG * b + cc;
            if (c >= nb) continue;
            if (tx == cc) {
#pragma unroll
                for (int a = 0; a < TS; ++a) {
                    const int i = ty + TG * a;
                    if (i < c) wb[buf][i] = M[a][b];
                    else if (i == c) {
                        // the pivot's owner: 1/sqrt(d) (hardware estimate refined by one
                        // Newton step), or NaN to flag a pivot <= 0 / NaN
                        const T d = M[a][b];
                        wb[buf][c] = T(-1);
                        T ip = T(NAN);
                        if (d > T(0) && isfinite((double)d)) {
                            ip = rsqrt(d);
                            ip = ip * (T(1.5) - T(0.5) * d * ip * ip);
                        }
                        dpiv[buf] = ip;
                    }
                }
            }
            if (ty == cc) {
#pragma unroll
                for (int b2 = 0; b2 < TS; ++b2) {
                    const int j = tx + TG * b2;
                    if (j > c && j < nb) wb[buf][j] = M[b][b2];
                }
            }
            __syncthreads();
            T ipiv = dpiv[buf];
            if (!(ipiv == ipiv)) {   // pivot <= 0 or NaN: report, go on with a unit pivot
                if (tid == 0) report(GPTQ_ERR_NOT_PD, col_base + c);
                ipiv = T(1);
            }
            T u[TS], v[TS];
#pragma unroll
            for (int a = 0; a < TS; ++a) {
                const int i = ty + TG * a;
                u[a] = i < c ? wb[buf][i] * ipiv : T(0);
            }
#pragma unroll
            for (int b2 = 0; b2 < TS; ++b2) {
                const int j = tx + TG * b2;
                v[b2] = j < nb ? -ipiv * wb[buf][j] : T(0);
            }
            if (tx == cc) {
#pragma unroll
                for (int a = 0; a < TS; ++a)
                    if (ty + TG * a < c) M[a][b] = T(0);
            }
#pragma unroll
            for (int a = 0; a < TS; ++a) {
                if (ty + TG * a < c) {
#pragma unroll
                    for (int b2 = 0; b2 < TS; ++b2) M[a][b2] = fma(u[a], v[b2], M[a][b2]);
                }
            }
            if (ty == cc) {
#pragma unroll
                for (int b2 = 0; b2 < TS; ++b2) {
                    const int j = tx + TG * b2;
                    if (j >= c && j < nb) M[b][b2] = v[b2];
                }
            }
            buf ^= 1;
        }
    }
#pragma unroll
    for (int a = 0; a < TS; ++a)
#pragma unroll
        for (int b = 0; b < TS; ++b) {
            const int i = ty + TG * a, j = tx + TG * b;
            if (i < nb && j < nb) U[(long long)i * ldu + j] = j >= i ? M[a][b] : T(0);
        }
}

// U_pp = inverse of the UL factor of the nb x nb block at A (nb <= FACTOR_NB).
template <typename T>
inline int diag_ul_inv(const T *A, long long lda, T *U, long long ldu, int nb, long long col_base,
                       cudaStream_t s, const int *skip = nullptr) {
    constexpr int TG = DiagCfg<T>::TG;
    return launch_kernel(diag_ul_inv_kernel<T>, dim3(1), dim3(TG * TG), 0, s, true, A, lda, U, ldu,
                         nb, col_base, skip);
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

// ---------------------------------------------------------------------------------------
// Leaf of the blocked factor, itself blocked (fp32): the 128 x 128 block is cut into four
// 32-column blocks, last first, and for block k (columns r .. r + 31) of the Schur
// complement S (shared memory, both triangles kept):
//   A  one warp: UL-Cholesky of S[k, k] and the inverse X_kk of its factor, in registers
//      (lane i holds row i). Step c needs the pivot column u = S[:c, c] / sqrt(d) and row c:
//      while the leading block is symmetric, row c also carries the pivot column
//      (S[c, j] = S[j, c] for j < c), so lane c's row is the only thing exchanged (one
//      shared-memory row per step) and every lane applies m_j += a r_j with one scalar a
//      (-u_i / sqrt(d) for rows above c, -1 - 1/sqrt(d) for row c itself, which turns its
//      entries right of c into row c of the inverse, 0 below). Registers rotate by one per
//      step so the pivot's register index is static and the loop body is one step;
//   B  Ubar's panel Ubar[0:r, k] = S[0:r, k] X_kk^T, written over S[0:r, k];
//   C  S[0:r, 0:r] -= Ubar[0:r, k] Ubar[0:r, k]^T;
//   D  X[k, >k] = -X_kk (Ubar[k, >k] X[>k, >k]): the inverse's rows right of the diagonal.
// A block with nb < 128 is padded with the identity (it couples to nothing).
// ---------------------------------------------------------------------------------------
constexpr int LB = 32;
constexpr int LB_LD = FACTOR_NB + 4;     // stride of S and X (16-byte rows)
constexpr int LB_TLD = FACTOR_NB - LB + 4;
constexpr int LEAF_THREADS = 256;
constexpr size_t LEAF_BLK_SMEM =
    sizeof(float) * (2 * (size_t)FACTOR_NB * LB_LD + (size_t)LB * LB_TLD + 2 * LB);
constexpr size_t LEAF_EXCLUSIVE_SMEM = 227 * 1024;  // the per-block maximum on sm_100
static_assert(LEAF_BLK_SMEM <= LEAF_EXCLUSIVE_SMEM, "leaf fits the exclusive allocation");

// A: X_kk of the 32 x 32 block of S at (r, r), written to X (warp 0 only). Before step c,
// physical register p holds column (p - 31 + c) mod 32, so the pivot is always m[31]; the
// rotation by one that keeps it there is folded into the update, and the loop body is one
// step (a short body also keeps the first, cold pass through the code cheap).
__device__ __forceinline__ void leaf_diag32_regs(float (&m)[LB], float *Xm, float *rowbuf, int r,
                                                 long long col_base, int i) {
#pragma unroll 1
    for (int c = LB - 1; c >= 0; --c) {
        float *rb = rowbuf + (c & 1) * LB;
        if (i == c) {
#pragma unroll
            for (int p4 = 0; p4 < LB; p4 += 4)
                *reinterpret_cast<float4 *>(rb + p4) = make_float4(m[p4], m[p4 + 1], m[p4 + 2], m[p4 + 3]);
        }
        const float d = __shfl_sync(0xffffffffu, m[LB - 1], c);
        const bool bad = !(d > 0.f) || !isfinite(d);
        if (bad && i == 0) report(GPTQ_ERR_NOT_PD, col_base + r + c);
        const float dd = bad ? 1.f : d;
        float ip = rsqrtf(dd);
        ip = ip * (1.5f - 0.5f * dd * ip * ip);  // one Newton step
        const float uu = m[LB - 1] * ip;
        const float a = i < c ? -uu * ip : (i == c ? -1.f - ip : 0.f);
        __syncwarp();
        // new_p = m_p + a r_p (p < 31), new_31 = the restarted pivot entry; m_{p+1} <- new_p
        const float piv = i < c ? uu * ip : ip;
        float prev = piv;
#pragma unroll
        for (int p4 = 0; p4 < LB - 4; p4 += 4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(rb + p4);
            const float n0 = fmaf(a, t4.x, m[p4]), n1 = fmaf(a, t4.y, m[p4 + 1]);
            const float n2 = fmaf(a, t4.z, m[p4 + 2]), n3 = fmaf(a, t4.w, m[p4 + 3]);
            m[p4] = prev; m[p4 + 1] = n0; m[p4 + 2] = n1; m[p4 + 3] = n2;
            prev = n3;
        }
        const float4 t4 = *reinterpret_cast<const float4 *>(rb + LB - 4);
        const float n0 = fmaf(a, t4.x, m[LB - 4]), n1 = fmaf(a, t4.y, m[LB - 3]);
        const float n2 = fmaf(a, t4.z, m[LB - 2]);
        m[LB - 4] = prev; m[LB - 3] = n0; m[LB - 2] = n1; m[LB - 1] = n2;
    }
#pragma unroll
    for (int j = 0; j < LB; ++j) Xm[(r + i) * LB_LD + r + j] = j >= i ? m[j] : 0.f;
}

__device__ __forceinline__ void leaf_diag32(float *Sm, float *Xm, float *rowbuf, int r,
                                            long long col_base, int i) {
    float m[LB];
#pragma unroll
    for (int j = 0; j < LB; ++j) m[j] = Sm[(r + i) * LB_LD + r + j];
    leaf_diag32_regs(m, Xm, rowbuf, r, col_base, i);
}

// B, C, D of block KB (r = 32 KB rows above it, q = 96 - r columns right of it), 8 warps.
template <int KB>
__device__ __forceinline__ void leaf_block_updates(float *Sm, float *Xm, float *Tm, int tid) {
    constexpr int r = KB * LB, q = FACTOR_NB - r - LB;
    const int lane = tid & 31, w = tid >> 5;
    // B (compute): rows w + 8 t of S[0:r, k] X_kk^T, column lane; D1: T = Ubar[k, >k] X[>k, >k]
    constexpr int BT = r / 8;
    float pb[BT > 0 ? BT : 1];
    if constexpr (r > 0) {
#pragma unroll
        for (int t = 0; t < BT; ++t) pb[t] = 0.f;
#pragma unroll 2
        for (int mm = 0; mm < LB; mm += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(Xm + (r + lane) * LB_LD + r + mm);
#pragma unroll
            for (int t = 0; t < BT; ++t) {
                const float4 sv = *reinterpret_cast<const float4 *>(Sm + (w + 8 * t) * LB_LD + r + mm);
                pb[t] += sv.x * x.x + sv.y * x.y + sv.z * x.z + sv.w * x.w;
            }
        }
    }
    if constexpr (q > 0) {
        constexpr int QH = q / 32;
        float acc[4][QH];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int h = 0; h < QH; ++h) acc[p][h] = 0.f;
#pragma unroll 4
        for (int mm = r + LB; mm < FACTOR_NB; ++mm) {
            float x[QH], sv[4];
#pragma unroll
            for (int h = 0; h < QH; ++h) x[h] = Xm[mm * LB_LD + r + LB + lane + 32 * h];
#pragma unroll
            for (int p = 0; p < 4; ++p) sv[p] = Sm[(r + w + 8 * p) * LB_LD + mm];
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < QH; ++h) acc[p][h] = fmaf(sv[p], x[h], acc[p][h]);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int h = 0; h < QH; ++h) Tm[(w + 8 * p) * LB_TLD + lane + 32 * h] = acc[p][h];
    }
    __syncthreads();
    // B (write) and D2: X[k, >k] = -X_kk T
    if constexpr (r > 0) {
#pragma unroll
        for (int t = 0; t < BT; ++t) Sm[(w + 8 * t) * LB_LD + r + lane] = pb[t];
    }
    if constexpr (q > 0) {
        constexpr int QH = q / 32;
        float acc[4][QH];
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int h = 0; h < QH; ++h) acc[p][h] = 0.f;
#pragma unroll 4
        for (int c2 = 0; c2 < LB; ++c2) {
            float x[4], tv[QH];
#pragma unroll
            for (int p = 0; p < 4; ++p) x[p] = Xm[(r + w + 8 * p) * LB_LD + r + c2];
#pragma unroll
            for (int h = 0; h < QH; ++h) tv[h] = Tm[c2 * LB_TLD + lane + 32 * h];
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < QH; ++h) acc[p][h] = fmaf(x[p], tv[h], acc[p][h]);
        }
#pragma unroll
        for (int p = 0; p < 4; ++p)
#pragma unroll
            for (int h = 0; h < QH; ++h) Xm[(r + w + 8 * p) * LB_LD + r + LB + lane + 32 * h] = -acc[p][h];
    }
    __syncthreads();
    // C: S[0:r, 0:r] -= P P^T, P = S[0:r, r:r+32]; thread (ty, tx) of 16 x 16 owns rows
    // ty + 16 a, columns tx + 16 b
    if constexpr (r > 0) {
        constexpr int CT = r / 16;
        const int tx = tid & 15, ty = tid >> 4;
        float acc[CT][CT];
#pragma unroll
        for (int a = 0; a < CT; ++a)
#pragma unroll
            for (int b = 0; b < CT; ++b) acc[a][b] = 0.f;
#pragma unroll 2
        for (int c = 0; c < LB; c += 4) {
            float4 pa[CT], pv[CT];
#pragma unroll
            for (int a = 0; a < CT; ++a) {
                pa[a] = *reinterpret_cast<const float4 *>(Sm + (ty + 16 * a) * LB_LD + r + c);
                pv[a] = *reinterpret_cast<const float4 *>(Sm + (tx + 16 * a) * LB_LD + r + c);
            }
#pragma unroll
            for (int a = 0; a < CT; ++a)
#pragma unroll
                for (int b = 0; b < CT; ++b)
                    acc[a][b] += pa[a].x * pv[b].x + pa[a].y * pv[b].y + pa[a].z * pv[b].z + pa[a].w * pv[b].w;
        }
#pragma unroll
        for (int a = 0; a < CT; ++a)
#pragma unroll
            for (int b = 0; b < CT; ++b) Sm[(ty + 16 * a) * LB_LD + tx + 16 * b] -= acc[a][b];
    }
    __syncthreads();
}

template <int KB>
__device__ __forceinline__ void leaf_block(float *Sm, float *Xm, float *Tm, float *rowbuf,
                                           long long col_base, int tid) {
    if (tid < 32) leaf_diag32(Sm, Xm, rowbuf, KB * LB, col_base, tid);
    __syncthreads();
    leaf_block_updates<KB>(Sm, Xm, Tm, tid);
}

__global__ __launch_bounds__(LEAF_THREADS) void leaf_blk_kernel(const float *A, long long lda,
                                                                float *U, long long ldu, int nb,
                                                                long long col_base) {
    extern __shared__ __align__(16) float lsm[];
    float *Sm = lsm;                                  // [128][132] Schur complement / panels
    float *Xm = Sm + FACTOR_NB * LB_LD;               // [128][132] the inverse (upper)
    float *Tm = Xm + FACTOR_NB * LB_LD;               // [32][100]  Ubar[k, >k] X[>k, >k]
    float *rowbuf = Tm + LB * LB_TLD;                 // [2][32]    row c of step c
    const int tid = threadIdx.x;
    pdl_wait_prev();
    constexpr int R3 = FACTOR_NB - LB;                // first column of the last 32-block
    if (tid < 32) {
        // warp 0 takes the last diagonal block straight from A and factors it while the other
        // warps stage the rest (its first, instruction-cache-cold pass overlaps the staging)
        float m[LB];
        const int i = R3 + tid;
#pragma unroll
        for (int jj = 0; jj < LB; ++jj) {
            const int j = R3 + jj;
            float v;
            if (i < nb && j < nb) v = j >= i ? A[(long long)i * lda + j] : A[(long long)j * lda + i];
            else v = i == j ? 1.f : 0.f;
            m[jj] = v;
        }
        leaf_diag32_regs(m, Xm, rowbuf, R3, col_base, tid);
    } else {
        // stage S symmetrically from A's upper triangle (coalesced rows); X starts at zero
        // except the block warp 0 writes
#pragma unroll 8
        for (int idx = tid - 32; idx < FACTOR_NB * FACTOR_NB; idx += LEAF_THREADS - 32) {
            const int i = idx >> 7, j = idx & (FACTOR_NB - 1);
            if (j >= i) {
                const float v = (i < nb && j < nb) ? A[(long long)i * lda + j] : (i == j ? 1.f : 0.f);
                Sm[i * LB_LD + j] = v;
                Sm[j * LB_LD + i] = v;
            }
            if (i < R3 || j < R3) Xm[i * LB_LD + j] = 0.f;
        }
    }
    __syncthreads();
    leaf_block_updates<3>(Sm, Xm, Tm, tid);
    leaf_block<2>(Sm, Xm, Tm, rowbuf, col_base, tid);
    leaf_block<1>(Sm, Xm, Tm, rowbuf, col_base, tid);
    leaf_block<0>(Sm, Xm, Tm, rowbuf, col_base, tid);
    pdl_launch_next();
#pragma unroll 4
    for (int idx = tid; idx < FACTOR_NB * FACTOR_NB; idx += LEAF_THREADS) {
        const int i = idx >> 7, j = idx & (FACTOR_NB - 1);
        if (i < nb && j < nb) U[(long long)i * ldu + j] = j >= i ? Xm[i * LB_LD + j] : 0.f;
    }
}

// pdl: launch as a programmatic dependent of the stream's previous kernel.
inline int leaf_ul_inv(const float *A, long long lda, float *U, long long ldu, int nb,
                       long long col_base, cudaStream_t s, bool pdl = false) {
    // GPTQ_LEAF=0 selects the barrier-synchronised leaf (diag_ul_inv_kernel)
    static const bool blocked = tc::env_ll("GPTQ_LEAF", 1) != 0;
    if (!blocked) return diag_ul_inv<float>(A, lda, U, ldu, nb, col_base, s);
    // With GPTQ_LEAF_EXCLUSIVE (default 1) the leaf asks for the whole of its SM's shared
    // memory, so that no CTA of the concurrent GEMMs lands beside it and takes its issue slots.
    static const bool exclusive = tc::env_ll("GPTQ_LEAF_EXCLUSIVE", 1) != 0;
    const size_t smem = exclusive ? LEAF_EXCLUSIVE_SMEM : LEAF_BLK_SMEM;
    GPTQ_SMEM_LIMIT(leaf_blk_kernel, smem);
    return launch_kernel(leaf_blk_kernel, dim3(1), dim3(LEAF_THREADS), smem, s, pdl, A,
                         lda, U, ldu, nb, col_base);
}

// Scratch of factor_ul_inverse, in blocks of FACTOR_NB x n floats: a copy of one row block of
// U, and the panel split into tf32 pairs for the trailing update.
constexpr int FACTOR_T_BLOCKS = 3;

// Lt[:, 0:cols] (rows x cols, row stride lda) split into tf32 pairs (round to nearest), row
// stride cols: the trailing update's operands, which then need no conversion.
__global__ void split_panel_kernel(const float *Lt, long long lda, int rows, int cols, float *Lh,
                                   float *Ll) {
    const long long total = (long long)rows * cols;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(idx / cols), j = (int)(idx % cols);
        const float v = Lt[(long long)i * lda + j];
        const float h = tcg::to_tf32(v);
        Lh[idx] = h;
        Ll[idx] = tcg::to_tf32(v - h);
    }
}

// Streams of the blocked factor: the pivot chain (leaf, and the two 128 x 128 products that
// feed the next leaf) on a high-priority stream; the rest of each panel and look-ahead column,
// the trailing update and the inverse's rows on three others. One set per device and slot,
// made on the first call; the mutex keeps the event protocol of one call intact against calls
// from other host threads.
struct FactorStreams {
    cudaStream_t chain = nullptr, panel = nullptr, bulk = nullptr, inv = nullptr;
    cudaEvent_t fork = nullptr, leaf_done = nullptr, pdiag_done = nullptr, prest_done = nullptr,
                larest_done = nullptr, bulk_done = nullptr, join[4] = {};
    std::mutex mu;
    bool ready = false;
};

// One set per device and slot: factorizations enqueued on different slots can run at once.
constexpr int FACTOR_SLOTS = 2;
inline FactorStreams *factor_streams(int slot) {
    static FactorStreams fs[64][FACTOR_SLOTS];
    static std::mutex init_mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (slot < 0 || slot >= FACTOR_SLOTS) return nullptr;
    std::lock_guard<std::mutex> lk(init_mu);
    FactorStreams &f = fs[dev][slot];
    if (!f.ready) {
        int lo = 0, hi = 0;
        cudaDeviceGetStreamPriorityRange(&lo, &hi);
        bool ok = cudaStreamCreateWithPriority(&f.chain, cudaStreamNonBlocking, hi) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&f.panel, cudaStreamNonBlocking, hi) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&f.bulk, cudaStreamNonBlocking, lo) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&f.inv, cudaStreamNonBlocking, lo) == cudaSuccess;
        cudaEvent_t *evs[] = {&f.fork, &f.leaf_done, &f.pdiag_done, &f.prest_done, &f.larest_done,
                              &f.bulk_done, &f.join[0], &f.join[1], &f.join[2], &f.join[3]};
        for (cudaEvent_t *e : evs)
            ok = ok && cudaEventCreateWithFlags(e, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return nullptr;
        f.ready = true;
    }
    return &f;
}

// Blocked right-looking UL factor with the inverse formed alongside (fp32, tensor-core
// GEMMs). A (n x n, lda) holds the damped matrix in its upper triangle on entry; its strictly
// lower block rows receive the panels transposed and the upper triangle is consumed. U (n x
// n, ldu) must be zero on entry and receives U = Ubar^-1, where A = Ubar Ubar^T, Ubar upper
// (so that A^-1 = U^T U with U upper: the factor the column sweep uses). With 128-column
// blocks k = K-1 .. 0, r = first column of block k, r1 = r - 128 (block k-1). T holds
// FACTOR_T_BLOCKS x 128 x n floats of scratch.
//   chain  X_kk  = leaf(A_kk)                                (Ubar_kk^-1)
//          L_k[k-1]^T = X_kk A[r1:r, k]^T                     (the panel's rows of block k-1)
//          A[r1:r, k-1] -= L_k[k-1] L_k[k-1]^T                (look-ahead: the next diagonal)
//   panel  L_k[0:r1]^T = X_kk A[0:r1, k]^T                    (the rest of the panel)
//          A[0:r1, k-1] -= L_k[0:r1] L_k[k-1]^T               (the rest of the look-ahead)
//   bulk   A[0:r1, 0:r1] -= L_k[0:r1] L_k[0:r1]^T              (upper triangle)
//   inv    U[k, >k] = -X_kk P[k, >k],  P[0:r, k:] += L_k U[k, k:]
// where P = U's upper part before its row block is final: P[i, j] = sum_l Ubar[i, l] X[l, j]
// over the finished row blocks l, from Ubar X = I. Only the chain is serial from block to
// block. Its products for block k-1 wait for the look-ahead rest of block k+1 (rows of block
// k-1 in column block k) and for the trailing update of block k+1 (which also writes the next
// diagonal block); the panel's look-ahead waits for that trailing update too (both write
// column block k-1).
inline int factor_ul_inverse(float *A, long long lda, float *U, long long ldu, int n, float *T,
                             cudaStream_t s, int slot = 0) {
    KtStageScope stage(GPTQ_KT_FACTOR);
    if (n <= FACTOR_NB) return leaf_ul_inv(A, lda, U, ldu, n, 0, s);
    FactorStreams *fs = factor_streams(slot);
    if (!fs) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(fs->mu);
    const int sms = device_sm_count();
    // persistent CTAs of the trailing update and of the inverse's GEMMs: the rest of the SMs
    // stay free for the chain and the panel stream
    static const long long side_env = tc::env_ll("GPTQ_FACTOR_SIDE_CTAS", 0);
    static const long long bulk_env = tc::env_ll("GPTQ_FACTOR_BULK_CTAS", 0);
    static const long long inv_env = tc::env_ll("GPTQ_FACTOR_INV_CTAS", 0);
    const int side = side_env > 0 ? (int)side_env : (2 * sms) / 3;
    const int bulk_ctas = bulk_env > 0 ? (int)bulk_env : side;
    const int inv_ctas = inv_env > 0 ? (int)inv_env : side;
    if (cudaEventRecord(fs->fork, s) != cudaSuccess) return GPTQ_ERR_CUDA;
    cudaStream_t streams[4] = {fs->chain, fs->panel, fs->bulk, fs->inv};
    for (cudaStream_t st2 : streams) cudaStreamWaitEvent(st2, fs->fork, 0);
    const int K = ceil_div(n, FACTOR_NB);
    int st = GPTQ_OK;
    for (int k = K - 1; k >= 0 && st == GPTQ_OK; --k) {
        const int r = k * FACTOR_NB, bk = std::min(FACTOR_NB, n - r);
        const int r1 = r - FACTOR_NB;  // first column of block k-1 (k > 0)
        float *Xkk = U + (long long)r * ldu + r;
        float *Lt = A + (long long)r * lda;  // L_k^T: bk x r, strict lower block row k
        // chain: the leaf starts while its predecessor (the last look-ahead) finishes
        if ((st = leaf_ul_inv(A + (long long)r * lda + r, lda, Xkk, ldu, bk, r, fs->chain, true))) break;
        cudaEventRecord(fs->leaf_done, fs->chain);
        if (k > 0) {
            // rows of block k-1 in column block k carry the look-ahead rest of block k+1
            if (k < K - 1) cudaStreamWaitEvent(fs->chain, fs->larest_done, 0);
            auto p = gemm_args<float, float>(bk, FACTOR_NB, bk, Xkk, ldu, 0,
                                             A + (long long)r1 * lda + r, lda, 1, Lt + r1, lda,
                                             1.f, 0.f);
            p.a_upper = 1;
            p.pdl = 1;
            if ((st = gemm_simt(p, fs->chain))) break;
            cudaEventRecord(fs->pdiag_done, fs->chain);
            // the next diagonal block, after the trailing update of block k+1 has written it
            if (k < K - 1) cudaStreamWaitEvent(fs->chain, fs->bulk_done, 0);
            auto q = gemm_args<float, float>(FACTOR_NB, FACTOR_NB, bk, Lt + r1, lda, 1, Lt + r1, lda,
                                             0, A + (long long)r1 * lda + r1, lda, -1.f, 1.f);
            q.pdl = 1;
            if ((st = gemm_simt(q, fs->chain))) break;
        }
        // panel: the rest of L_k and of the look-ahead column
        if (k > 1) {
            cudaStreamWaitEvent(fs->panel, fs->leaf_done, 0);
            auto p = gemm_args<float, float>(bk, r1, bk, Xkk, ldu, 0, A + r, lda, 1, Lt, lda, 1.f, 0.f);
            p.a_upper = 1;
            p.pdl = 1;
            if ((st = gemm_simt(p, fs->panel))) break;
            cudaEventRecord(fs->prest_done, fs->panel);
            cudaStreamWaitEvent(fs->panel, fs->pdiag_done, 0);
            if (k < K - 1) cudaStreamWaitEvent(fs->panel, fs->bulk_done, 0);
            auto q = gemm_args<float, float>(r1, FACTOR_NB, bk, Lt, lda, 1, Lt + r1, lda, 0, A + r1,
                                             lda, -1.f, 1.f);
            q.pdl = 1;
            if ((st = gemm_simt(q, fs->panel))) break;
            cudaEventRecord(fs->larest_done, fs->panel);
            // bulk: the trailing update of everything left of block k-1, from the panel split
            // once into tf32 pairs (both operands are L_k)
            cudaStreamWaitEvent(fs->bulk, fs->prest_done, 0);
            float *Lh = T + (size_t)FACTOR_NB * n, *Ll = Lh + (size_t)FACTOR_NB * n;
            const bool split = r1 >= 256 && r1 % 4 == 0 && (reinterpret_cast<uintptr_t>(Lh) & 15u) == 0;
            if (split) {
                split_panel_kernel<<<2 * sms, 256, 0, fs->bulk>>>(Lt, lda, bk, r1, Lh, Ll);
                if ((st = launch_status())) break;
            }
            auto b2 = split ? gemm_args<float, float>(r1, r1, bk, Lh, r1, 1, Lh, r1, 0, A, lda, -1.f, 1.f)
                            : gemm_args<float, float>(r1, r1, bk, Lt, lda, 1, Lt, lda, 0, A, lda, -1.f, 1.f);
            if (split) {
                b2.a_lo = Ll;
                b2.b_lo = Ll;
                b2.b_full = Lt;
                b2.ldb_full = lda;
            }
            b2.c_upper = 1;
            b2.max_ctas = bulk_ctas;
            if ((st = gemm_f32(b2, fs->bulk))) break;
            cudaEventRecord(fs->bulk_done, fs->bulk);
        }
        // inverse rows: need X_kk and the whole panel L_k
        cudaStreamWaitEvent(fs->inv, fs->leaf_done, 0);
        if (k > 0) {
            cudaStreamWaitEvent(fs->inv, fs->pdiag_done, 0);
            if (k > 1) cudaStreamWaitEvent(fs->inv, fs->prest_done, 0);
        }
        if (k < K - 1) {
            const int e = r + bk, wdt = n - e;
            float *row = U + (long long)r * ldu + e;
            if (cudaMemcpy2DAsync(T, sizeof(float) * wdt, row, sizeof(float) * ldu,
                                  sizeof(float) * wdt, bk, cudaMemcpyDeviceToDevice,
                                  fs->inv) != cudaSuccess) {
                st = GPTQ_ERR_CUDA;
                break;
            }
            auto p = gemm_args<float, float>(bk, wdt, bk, Xkk, ldu, 0, T, wdt, 0, row, ldu, -1.f, 0.f);
            p.a_upper = 1;
            p.max_ctas = inv_ctas;
            if ((st = gemm_f32(p, fs->inv))) break;
        }
        if (k > 0) {
            auto p = gemm_args<float, float>(r, n - r, bk, Lt, lda, 1, Xkk, ldu, 0, U + r, ldu, 1.f, 1.f);
            p.max_ctas = inv_ctas;
            if ((st = gemm_f32(p, fs->inv))) break;
        }
    }
    // join all four streams back into the caller's stream, on success and on error alike
    for (int i = 0; i < 4; ++i) {
        cudaEventRecord(fs->join[i], streams[i]);
        cudaStreamWaitEvent(s, fs->join[i], 0);
    }
    if (st == GPTQ_OK && cudaGetLastError() != cudaSuccess) st = GPTQ_ERR_CUDA;
    return st;
}

}  // namespace gptq
