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

// ---------------------------------------------------------------------------------------
// Leaf of the blocked factor (fp32): the same UL sweep as diag_ul_inv_kernel, organised so
// that no step waits on a CTA-wide barrier. Warp w owns the 16 columns 16w..16w+15; lane l
// holds rows l, l+32, l+64, l+96 of them (64 registers). Step c belongs to the warp that
// owns column c: it takes the pivot, publishes u = M[:c, c] / sqrt(d) and 1/sqrt(d) to
// shared memory (one slot per step, written once) and its 32 lanes arrive on the step's
// mbarrier (release). Every other warp waits on that barrier (acquire; the hardware parks
// the waiting threads) and applies the step to its own columns: the Cholesky update
// (v_j = -u_j) left of c, the inverse update (v_j = -P[c][j] / sqrt(d), row c read from the
// lane that holds it) right of c.
//   Row c is final after step c (row c of the inverse, columns >= c): it goes to shared
// memory and its registers are dead, as are all rows below it, so step c only touches the
// row slots that still hold rows < c. During its 16 steps the owner rotates its columns by
// one register position per step (the update of position p lands in p + 1, the restarted
// pivot column in 0), so the pivot is always in position 15 and every register index is a
// compile-time constant; 16 rotations restore the order. Only the loop over the 4 row slots
// is unrolled, which keeps the code each warp runs within the instruction cache.
// ---------------------------------------------------------------------------------------
constexpr int LEAF_THREADS = 256;
constexpr int LEAF_LD = FACTOR_NB + 1;  // padded stride of the staging tile
constexpr size_t LEAF_SMEM = sizeof(float) * (2 * (size_t)FACTOR_NB * FACTOR_NB + FACTOR_NB);
static_assert(FACTOR_NB * LEAF_LD <= 2 * FACTOR_NB * FACTOR_NB, "staging fits the step slots");

template <int RC>
__device__ __forceinline__ void leaf_rotate(float (&M)[4][16]) {
#pragma unroll
    for (int r = 0; r <= RC; ++r) {
        const float t = M[r][15];
#pragma unroll
        for (int p = 14; p >= 0; --p) M[r][p + 1] = M[r][p];
        M[r][0] = t;
    }
}

// Steps c = 32 RC + 31 .. 32 RC of the sweep (rows of slot RC).
template <int RC>
__device__ __forceinline__ void leaf_slot_steps(float (&M)[4][16], float *pub, float *xrow,
                                                float *pipiv, uint64_t *step_bar, int nb,
                                                long long col_base, long long wait_limit,
                                                int lane, int w, bool &stop) {
#pragma unroll 1
    for (int cc = 31; cc >= 0; --cc) {
        const int c = 32 * RC + cc, ob = c >> 4, s = 15 - (c & 15);
        if (stop) return;
        if (c >= nb) {
            if (w == ob) leaf_rotate<RC>(M);  // keep the owner's rotation count
            continue;
        }
        float u[RC + 1], v[16];
        if (w == ob) {
            const float d = __shfl_sync(0xffffffffu, M[RC][15], cc);
            const bool bad = !(d > 0.f) || !isfinite(d);
            if (bad && lane == 0) report(GPTQ_ERR_NOT_PD, col_base + c);
            const float dd = bad ? 1.f : d;
            float ipiv = rsqrtf(dd);
            ipiv = ipiv * (1.5f - 0.5f * dd * ipiv * ipiv);  // one Newton step
#pragma unroll
            for (int r = 0; r <= RC; ++r) {
                u[r] = (r < RC || lane < cc) ? M[r][15] * ipiv : 0.f;
                pub[c * FACTOR_NB + lane + 32 * r] = u[r];
            }
            if (lane == 0) pipiv[c] = ipiv;
            tc::mbar_arrive(&step_bar[c]);
            // position p holds column 16 ob + ((p - s) mod 16): p < s right of c, s <= p < 15
            // left of c (its u sits in lane (16 ob + p - s) mod 32 of this slot)
            const int jl = (16 * ob - s) & 31;
#pragma unroll
            for (int p = 0; p < 15; ++p) {
                const float a = __shfl_sync(0xffffffffu, M[RC][p], cc);
                const float b = __shfl_sync(0xffffffffu, u[RC], (jl + p) & 31);
                v[p] = p < s ? -ipiv * a : -b;
            }
            v[15] = ipiv;
            if (lane == cc) {
#pragma unroll
                for (int p = 0; p < 16; ++p)
                    if (p < s || p == 15) xrow[c * FACTOR_NB + 16 * ob + ((p - s) & 15)] = v[p];
            }
#pragma unroll
            for (int r = 0; r <= RC; ++r) {
#pragma unroll
                for (int p = 14; p >= 0; --p) M[r][p + 1] = fmaf(u[r], v[p], M[r][p]);
                M[r][0] = u[r] * ipiv;
            }
        } else {
            if (!tc::mbar_wait(&step_bar[c], 0u, wait_limit)) {
                if (lane == 0) report(GPTQ_ERR_TIMEOUT, col_base + c);
                stop = true;
                return;
            }
            const float ipiv = pipiv[c];
#pragma unroll
            for (int r = 0; r <= RC; ++r) u[r] = pub[c * FACTOR_NB + lane + 32 * r];
            if (w < ob) {
                const float4 *q = reinterpret_cast<const float4 *>(pub + c * FACTOR_NB + 16 * w);
#pragma unroll
                for (int b4 = 0; b4 < 4; ++b4) {
                    const float4 x = q[b4];
                    v[4 * b4 + 0] = -x.x; v[4 * b4 + 1] = -x.y;
                    v[4 * b4 + 2] = -x.z; v[4 * b4 + 3] = -x.w;
                }
            } else {
#pragma unroll
                for (int b = 0; b < 16; ++b) v[b] = -ipiv * __shfl_sync(0xffffffffu, M[RC][b], cc);
                if (lane == cc) {
                    float4 *q = reinterpret_cast<float4 *>(xrow + c * FACTOR_NB + 16 * w);
#pragma unroll
                    for (int b4 = 0; b4 < 4; ++b4)
                        q[b4] = make_float4(v[4 * b4], v[4 * b4 + 1], v[4 * b4 + 2], v[4 * b4 + 3]);
                }
            }
#pragma unroll
            for (int r = 0; r <= RC; ++r)
#pragma unroll
                for (int b = 0; b < 16; ++b) M[r][b] = fmaf(u[r], v[b], M[r][b]);
        }
    }
}

__global__ __launch_bounds__(LEAF_THREADS) void leaf_ul_inv_kernel(const float *A, long long lda,
                                                                   float *U, long long ldu, int nb,
                                                                   long long col_base,
                                                                   long long wait_limit) {
    extern __shared__ __align__(16) float leaf_sm[];
    float *stage = leaf_sm;                              // [128][LEAF_LD], before the sweep
    float *pub = leaf_sm;                                // [128][128]: u of step c at pub[128 c]
    float *xrow = leaf_sm + FACTOR_NB * FACTOR_NB;       // [128][128]: rows of the inverse
    float *pipiv = leaf_sm + 2 * FACTOR_NB * FACTOR_NB;  // [128]
    __shared__ uint64_t step_bar[FACTOR_NB];             // one single-use barrier per step
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

    // stage the block symmetrically from its upper triangle (coalesced rows)
#pragma unroll 8
    for (int idx = tid; idx < FACTOR_NB * FACTOR_NB; idx += LEAF_THREADS) {
        const int i = idx >> 7, j = idx & (FACTOR_NB - 1);
        const float v = (j >= i && i < nb && j < nb) ? A[(long long)i * lda + j] : 0.f;
        if (j >= i) {
            stage[i * LEAF_LD + j] = v;
            stage[j * LEAF_LD + i] = v;
        }
    }
    if (tid < FACTOR_NB) tc::mbar_init(&step_bar[tid], 32);
    __syncthreads();
    float M[4][16];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int b = 0; b < 16; ++b) M[r][b] = stage[(lane + 32 * r) * LEAF_LD + 16 * w + b];
    __syncthreads();

    bool stop = false;
    leaf_slot_steps<3>(M, pub, xrow, pipiv, step_bar, nb, col_base, wait_limit, lane, w,
                       stop);
    leaf_slot_steps<2>(M, pub, xrow, pipiv, step_bar, nb, col_base, wait_limit, lane, w,
                       stop);
    leaf_slot_steps<1>(M, pub, xrow, pipiv, step_bar, nb, col_base, wait_limit, lane, w,
                       stop);
    leaf_slot_steps<0>(M, pub, xrow, pipiv, step_bar, nb, col_base, wait_limit, lane, w,
                       stop);
    __syncthreads();
#pragma unroll 8
    for (int idx = tid; idx < FACTOR_NB * FACTOR_NB; idx += LEAF_THREADS) {
        const int i = idx >> 7, j = idx & (FACTOR_NB - 1);
        if (i < nb && j < nb) U[(long long)i * ldu + j] = j >= i ? xrow[i * FACTOR_NB + j] : 0.f;
    }
}

// ---------------------------------------------------------------------------------------
// Leaf of the blocked factor, itself blocked (fp32): the 128 x 128 block is cut into four
// 32-column blocks, last first, and for block k (columns r .. r + 31) of the Schur
// complement S (shared memory, both triangles kept):
//   A  one warp: UL-Cholesky of S[k, k] and the inverse X_kk of its factor, in registers
//      (lane i holds row i; the column sweep of the barrier leaf, with its row and column
//      exchanged through shared memory inside the warp);
//   B  Ubar's panel Ubar[0:r, k] = S[0:r, k] X_kk^T, written over S[0:r, k];
//   C  S[0:r, 0:r] -= Ubar[0:r, k] Ubar[0:r, k]^T;
//   D  X[k, >k] = -X_kk (Ubar[k, >k] X[>k, >k]): the inverse's rows right of the diagonal.
// A block with nb < 128 is padded with the identity (it couples to nothing). Only the
// diagonal steps of A are sequential; B, C and D are small products over all 8 warps.
// ---------------------------------------------------------------------------------------
constexpr int LB = 32;
constexpr int LB_LD = FACTOR_NB + 1;     // padded stride of S and X
constexpr int LB_TLD = FACTOR_NB - LB + 1;
constexpr size_t LEAF_BLK_SMEM =
    sizeof(float) * (2 * (size_t)FACTOR_NB * LB_LD + (size_t)LB * LB_TLD + 4 * LB);

__global__ __launch_bounds__(LEAF_THREADS) void leaf_blk_kernel(const float *A, long long lda,
                                                                float *U, long long ldu, int nb,
                                                                long long col_base) {
    extern __shared__ __align__(16) float lsm[];
    float *Sm = lsm;                                  // [128][129] Schur complement / panels
    float *Xm = Sm + FACTOR_NB * LB_LD;               // [128][129] the inverse (upper)
    float *Tm = Xm + FACTOR_NB * LB_LD;               // [32][97]   Ubar[k, >k] X[>k, >k]
    float *xb = Tm + LB * LB_TLD;                     // [2][2][32] step exchange (u, row c)
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;

#pragma unroll 4
    for (int idx = tid; idx < FACTOR_NB * FACTOR_NB; idx += LEAF_THREADS) {
        const int i = idx >> 7, j = idx & (FACTOR_NB - 1);
        float v;
        if (i < nb && j < nb) v = j >= i ? A[(long long)i * lda + j] : A[(long long)j * lda + i];
        else v = i == j ? 1.f : 0.f;
        Sm[i * LB_LD + j] = v;
        Xm[i * LB_LD + j] = 0.f;
    }
    __syncthreads();

#pragma unroll 1
    for (int kb = FACTOR_NB / LB - 1; kb >= 0; --kb) {
        const int r = kb * LB;
        const int q = FACTOR_NB - r - LB;             // columns right of block k
        // ---- A: the diagonal block -------------------------------------------------------
        if (w == 0) {
            const int i = lane;
            float m[LB];
#pragma unroll
            for (int j = 0; j < LB; ++j) m[j] = Sm[(r + i) * LB_LD + r + j];
#pragma unroll
            for (int c = LB - 1; c >= 0; --c) {
                float *ub = xb + (c & 1) * 2 * LB, *rb = ub + LB;
                const float d = __shfl_sync(0xffffffffu, m[c], c);
                const bool bad = !(d > 0.f) || !isfinite(d);
                if (bad && i == 0) report(GPTQ_ERR_NOT_PD, col_base + r + c);
                const float dd = bad ? 1.f : d;
                float ip = rsqrtf(dd);
                ip = ip * (1.5f - 0.5f * dd * ip * ip);  // one Newton step
                const float u = i < c ? m[c] * ip : 0.f;
                ub[i] = -u;
                if (i == c) {
#pragma unroll
                    for (int j = c + 1; j < LB; ++j) rb[j] = -ip * m[j];
                }
                __syncwarp();
                if (i == c) {
                    m[c] = ip;
#pragma unroll
                    for (int j = c + 1; j < LB; ++j) m[j] = rb[j];
                } else {
#pragma unroll
                    for (int j = 0; j < c; ++j) m[j] = fmaf(u, ub[j], m[j]);
                    m[c] = u * ip;
#pragma unroll
                    for (int j = c + 1; j < LB; ++j) m[j] = fmaf(u, rb[j], m[j]);
                }
            }
#pragma unroll
            for (int j = 0; j < LB; ++j) Xm[(r + i) * LB_LD + r + j] = j >= i ? m[j] : 0.f;
        }
        __syncthreads();
        // ---- B (compute) and D1 ----------------------------------------------------------
        float pb[12];
        if (r > 0) {
#pragma unroll
            for (int t = 0; t < 12; ++t) pb[t] = 0.f;
            const int c = lane;
#pragma unroll 4
            for (int mm = 0; mm < LB; ++mm) {
                const float x = Xm[(r + c) * LB_LD + r + mm];
#pragma unroll
                for (int t = 0; t < 12; ++t)
                    if (w + 8 * t < r) pb[t] = fmaf(Sm[(w + 8 * t) * LB_LD + r + mm], x, pb[t]);
            }
        }
        if (q > 0) {
            float acc[4][3];
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < 3; ++h) acc[p][h] = 0.f;
            for (int mm = r + LB; mm < FACTOR_NB; ++mm) {
                float x[3], sv[4];
#pragma unroll
                for (int h = 0; h < 3; ++h) {
                    const int jj = lane + 32 * h;
                    x[h] = jj < q ? Xm[mm * LB_LD + r + LB + jj] : 0.f;
                }
#pragma unroll
                for (int p = 0; p < 4; ++p) sv[p] = Sm[(r + w + 8 * p) * LB_LD + mm];
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int h = 0; h < 3; ++h) acc[p][h] = fmaf(sv[p], x[h], acc[p][h]);
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < 3; ++h) {
                    const int jj = lane + 32 * h;
                    if (jj < q) Tm[(w + 8 * p) * LB_TLD + jj] = acc[p][h];
                }
        }
        __syncthreads();
        // ---- B (write) and D2 ------------------------------------------------------------
        if (r > 0) {
#pragma unroll
            for (int t = 0; t < 12; ++t)
                if (w + 8 * t < r) Sm[(w + 8 * t) * LB_LD + r + lane] = pb[t];
        }
        if (q > 0) {
            float acc[4][3];
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < 3; ++h) acc[p][h] = 0.f;
#pragma unroll 4
            for (int c2 = 0; c2 < LB; ++c2) {
                float x[4], tv[3];
#pragma unroll
                for (int p = 0; p < 4; ++p) x[p] = Xm[(r + w + 8 * p) * LB_LD + r + c2];
#pragma unroll
                for (int h = 0; h < 3; ++h) {
                    const int jj = lane + 32 * h;
                    tv[h] = jj < q ? Tm[c2 * LB_TLD + jj] : 0.f;
                }
#pragma unroll
                for (int p = 0; p < 4; ++p)
#pragma unroll
                    for (int h = 0; h < 3; ++h) acc[p][h] = fmaf(x[p], tv[h], acc[p][h]);
            }
#pragma unroll
            for (int p = 0; p < 4; ++p)
#pragma unroll
                for (int h = 0; h < 3; ++h) {
                    const int jj = lane + 32 * h;
                    if (jj < q) Xm[(r + w + 8 * p) * LB_LD + r + LB + jj] = -acc[p][h];
                }
        }
        __syncthreads();
        // ---- C: the Schur complement -----------------------------------------------------
        if (r > 0) {
            const int tx = tid & 15, ty = tid >> 4;
            float acc[6][6];
#pragma unroll
            for (int a = 0; a < 6; ++a)
#pragma unroll
                for (int b = 0; b < 6; ++b) acc[a][b] = 0.f;
#pragma unroll 2
            for (int c = 0; c < LB; ++c) {
                float pa[6], pbv[6];
#pragma unroll
                for (int a = 0; a < 6; ++a) {
                    pa[a] = ty + 16 * a < r ? Sm[(ty + 16 * a) * LB_LD + r + c] : 0.f;
                    pbv[a] = tx + 16 * a < r ? Sm[(tx + 16 * a) * LB_LD + r + c] : 0.f;
                }
#pragma unroll
                for (int a = 0; a < 6; ++a)
#pragma unroll
                    for (int b = 0; b < 6; ++b) acc[a][b] = fmaf(pa[a], pbv[b], acc[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 6; ++a)
#pragma unroll
                for (int b = 0; b < 6; ++b) {
                    const int i = ty + 16 * a, j = tx + 16 * b;
                    if (i < r && j < r) Sm[i * LB_LD + j] -= acc[a][b];
                }
        }
        __syncthreads();
    }
#pragma unroll 4
    for (int idx = tid; idx < FACTOR_NB * FACTOR_NB; idx += LEAF_THREADS) {
        const int i = idx >> 7, j = idx & (FACTOR_NB - 1);
        if (i < nb && j < nb) U[(long long)i * ldu + j] = j >= i ? Xm[i * LB_LD + j] : 0.f;
    }
}

inline int leaf_ul_inv(const float *A, long long lda, float *U, long long ldu, int nb,
                       long long col_base, cudaStream_t s) {
    // GPTQ_LEAF: 0 the barrier-synchronised leaf (diag_ul_inv_kernel), 1 (default) the
    // warp-owner leaf, 2 the blocked leaf
    static const long long leaf = tc::env_ll("GPTQ_LEAF", 1);
    if (leaf == 0) return diag_ul_inv<float>(A, lda, U, ldu, nb, col_base, s);
    if (leaf == 2) {
        cudaFuncSetAttribute(leaf_blk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)LEAF_BLK_SMEM);
        leaf_blk_kernel<<<1, LEAF_THREADS, LEAF_BLK_SMEM, s>>>(A, lda, U, ldu, nb, col_base);
        return launch_status();
    }
    cudaFuncSetAttribute(leaf_ul_inv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)LEAF_SMEM);
    // clock cycles a warp waits for a step before the kernel gives up with GPTQ_ERR_TIMEOUT
    static const long long limit = tc::env_ll("GPTQ_WAIT_LIMIT_CYCLES", 4000000000LL);
    leaf_ul_inv_kernel<<<1, LEAF_THREADS, LEAF_SMEM, s>>>(A, lda, U, ldu, nb, col_base, limit);
    return launch_status();
}

// Streams of the blocked factor: the pivot chain (leaf, panel solve, look-ahead column) on a
// high-priority stream, the trailing update and the inverse's rows on two others. One set per
// device, made on the first call; the mutex keeps the event protocol of one call intact
// against calls from other host threads.
struct FactorStreams {
    cudaStream_t chain = nullptr, bulk = nullptr, inv = nullptr;
    cudaEvent_t fork = nullptr, panel = nullptr, bulk_done = nullptr, join[3] = {};
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
                  cudaStreamCreateWithPriority(&f.bulk, cudaStreamNonBlocking, lo) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&f.inv, cudaStreamNonBlocking, lo) == cudaSuccess;
        cudaEvent_t *evs[] = {&f.fork, &f.panel, &f.bulk_done, &f.join[0], &f.join[1], &f.join[2]};
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
// blocks k = K-1 .. 0, r = first column of block k:
//   chain  X_kk  = leaf(A_kk)                              (Ubar_kk^-1)
//          L_k^T = X_kk A[0:r, k]^T                         (panel of Ubar, kept transposed)
//          A[0:r, k-1] -= L_k L_k[k-1]^T                    (look-ahead: the next panel)
//   bulk   A[0:r', 0:r'] -= L_k L_k^T on r' = start of block k-1 (upper triangle)
//   inv    U[k, >k] = -X_kk P[k, >k],  P[0:r, k:] += L_k U[k, k:]
// where P = U's upper part before its row block is final: P[i, j] = sum_l Ubar[i, l] X[l, j]
// over the finished row blocks l, from Ubar X = I. The chain waits for the bulk update of
// the previous block before its look-ahead; the inverse stream trails both.
inline int factor_ul_inverse(float *A, long long lda, float *U, long long ldu, int n, float *T,
                             cudaStream_t s, int slot = 0) {
    if (n <= FACTOR_NB) return leaf_ul_inv(A, lda, U, ldu, n, 0, s);
    FactorStreams *fs = factor_streams(slot);
    if (!fs) return GPTQ_ERR_CUDA;
    std::lock_guard<std::mutex> lk(fs->mu);
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // persistent CTAs of each side-stream GEMM: the rest of the SMs stay free for the chain
    static const long long side_env = tc::env_ll("GPTQ_FACTOR_SIDE_CTAS", 0);
    const int side = side_env > 0 ? (int)side_env : (2 * sms) / 3;
    if (cudaEventRecord(fs->fork, s) != cudaSuccess) return GPTQ_ERR_CUDA;
    cudaStreamWaitEvent(fs->chain, fs->fork, 0);
    cudaStreamWaitEvent(fs->bulk, fs->fork, 0);
    cudaStreamWaitEvent(fs->inv, fs->fork, 0);
    const int K = ceil_div(n, FACTOR_NB);
    int st = GPTQ_OK;
    for (int k = K - 1; k >= 0 && st == GPTQ_OK; --k) {
        const int r = k * FACTOR_NB, bk = std::min(FACTOR_NB, n - r);
        float *Xkk = U + (long long)r * ldu + r;
        float *Lt = A + (long long)r * lda;  // L_k^T: bk x r, strict lower block row k
        if ((st = leaf_ul_inv(A + (long long)r * lda + r, lda, Xkk, ldu, bk, r, fs->chain))) break;
        if (k > 0) {
            auto p = gemm_args<float, float>(bk, r, bk, Xkk, ldu, 0, A + r, lda, 1, Lt, lda, 1.f, 0.f);
            p.a_upper = 1;
            // the chain's products are small (K = 128, at most 47 output tiles of 128): the SIMT
            // kernel's 64-tiles start sooner and spread wider than the tensor-core pipeline
            if ((st = gemm_simt(p, fs->chain))) break;
        }
        cudaEventRecord(fs->panel, fs->chain);
        if (k > 0) {
            const int r1 = r - FACTOR_NB;
            cudaStreamWaitEvent(fs->chain, fs->bulk_done, 0);  // bulk update of block k+1
            auto p = gemm_args<float, float>(r, FACTOR_NB, bk, Lt, lda, 1, Lt + r1, lda, 0, A + r1,
                                             lda, -1.f, 1.f);
            if ((st = gemm_simt(p, fs->chain))) break;
            if (r1 > 0) {
                cudaStreamWaitEvent(fs->bulk, fs->panel, 0);
                auto q = gemm_args<float, float>(r1, r1, bk, Lt, lda, 1, Lt, lda, 0, A, lda, -1.f, 1.f);
                q.c_upper = 1;
                q.max_ctas = side;
                if ((st = gemm_f32(q, fs->bulk))) break;
                cudaEventRecord(fs->bulk_done, fs->bulk);
            }
        }
        cudaStreamWaitEvent(fs->inv, fs->panel, 0);
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
            p.max_ctas = side;
            if ((st = gemm_f32(p, fs->inv))) break;
        }
        if (k > 0) {
            auto p = gemm_args<float, float>(r, n - r, bk, Lt, lda, 1, Xkk, ldu, 0, U + r, ldu, 1.f, 1.f);
            p.max_ctas = side;
            if ((st = gemm_f32(p, fs->inv))) break;
        }
    }
    // join all three streams back into the caller's stream, on success and on error alike
    cudaEventRecord(fs->join[0], fs->chain);
    cudaEventRecord(fs->join[1], fs->bulk);
    cudaEventRecord(fs->join[2], fs->inv);
    for (int i = 0; i < 3; ++i) cudaStreamWaitEvent(s, fs->join[i], 0);
    if (st == GPTQ_OK && cudaGetLastError() != cudaSuccess) st = GPTQ_ERR_CUDA;
    return st;
}

}  // namespace gptq
