// GPTQ-intrinsic LoRA on the device.
//
// GPTQ-intrinsic LoRA summary, "Method" part 2: X~ = [X, X V_r] with V_r the top-r right
// singular vectors of X; the pass runs on W~ = [W, 0]; the r extra coordinates absorb the
// error and become R; the singular augmented Hessian is factored without a plain Cholesky.
//
// Device route:
//   1. V_r: block subspace iteration on H (= 2 X^T X, same eigenvectors as X^T X) with
//      CholeskyQR2 re-orthonormalisation, then a Rayleigh-Ritz step whose small p x p
//      eigenproblem is solved by a one-CTA parallel-order Jacobi sweep.
//   2. H~ = [[H + l I, H V], [V^T H, V^T H V + l I]] with l = lambda_rel * mean of
//      its n + r raw diagonal entries. The first n rows of U~ (H~^-1 = U~^T U~) are
//      [U11, U12] with U11 the factor of the Schur complement S = H + l I - H V C^-1 V^T H
//      (C = V^T H V + l I) and U12 = -U11 H V C^-1. S is positive definite although H~ is
//      singular up to l, so the plain blocked factor applies to it.
//   3. The sweep on [W, 0] with those n rows; R = the final extra columns, transposed.
#pragma once

#include <utility>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "factor.cuh"

namespace gptq {

constexpr int IL_MAX_R = 128;

inline int il_block_p(int n, int r) {
    int p = r + 32 > 2 * r ? r + 32 : 2 * r;
    if (p > 128) p = 128;
    if (p > n) p = n;
    if (p & 1) p -= 1;
    if (p < r) p = r;  // only when n == r (odd): p = r
    return p;
}

__device__ __forceinline__ unsigned long long splitmix64(unsigned long long x) {
    x += 0x9E3779B97F4A7C15ull;
    x = (x ^ (x >> 30)) * 0xBF58476D1CE4E5B9ull;
    x = (x ^ (x >> 27)) * 0x94D049BB133111EBull;
    return x ^ (x >> 31);
}

// Deterministic start block: entries uniform in (-1, 1) from a counter hash.
__global__ void random_block_kernel(float *Y, long long total, unsigned long long seed) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const unsigned long long h = splitmix64(seed ^ (unsigned long long)i * 0xD1B54A32D192ED03ull);
        Y[i] = (float)((double)(h >> 11) * (2.0 / 9007199254740992.0) - 1.0);
    }
}

// One-CTA cyclic Jacobi on a symmetric p x p matrix (p even, p <= 128), round-robin
// ordering so that p/2 disjoint rotations run at once. The matrix is held in fp64, the
// accumulated rotations in fp32 (both in shared memory). On exit the r largest eigenvalues
// are written in decreasing order to evals[0..r) and their eigenvectors to the columns of
// Qsel (p x r).
__global__ __launch_bounds__(512) void jacobi_eig_kernel(const double *Tin, int p, int r,
                                                         float *Qsel, double *evals) {
    extern __shared__ __align__(16) unsigned char jsm[];
    const int LD = p + 1;
    double *T = reinterpret_cast<double *>(jsm);
    double *cs = T + p * LD;      // p/2 cosines
    double *sn = cs + p / 2;      // p/2 sines
    float *Q = reinterpret_cast<float *>(sn + p / 2);
    int *pi = reinterpret_cast<int *>(Q + p * LD);
    int *pj = pi + p / 2;
    __shared__ double red[2];
    const int tid = threadIdx.x, nt = blockDim.x;
    const int warp = tid >> 5, lane = tid & 31, nwarps = nt >> 5;
    for (int idx = tid; idx < p * p; idx += nt) {
        const int i = idx / p, j = idx % p;
        T[i * LD + j] = 0.5 * (Tin[i * p + j] + Tin[j * p + i]);
        Q[i * LD + j] = (i == j) ? 1.f : 0.f;
    }
    const int half = p / 2;
    for (int sweep = 0; sweep < 20; ++sweep) {
        if (tid < 2) red[tid] = 0.0;
        __syncthreads();
        double off = 0.0, dia = 0.0;
        for (int idx = tid; idx < p * p; idx += nt) {
            const int i = idx / p, j = idx % p;
            const double v = T[i * LD + j];
            if (i != j) off += v * v; else dia += v * v;
        }
        off = warp_sum_d(off);
        dia = warp_sum_d(dia);
        if ((tid & 31) == 0) { atomicAdd(&red[0], off); atomicAdd(&red[1], dia); }
        __syncthreads();
        const bool done = red[0] <= 1e-26 * red[1];
        __syncthreads();
        if (done) break;
        for (int rnd = 0; rnd < p - 1; ++rnd) {
            for (int k = tid; k < half; k += nt) {
                const int xb = p - 1 - k;
                const int a = k == 0 ? 0 : 1 + (k - 1 + rnd) % (p - 1);
                const int b = 1 + (xb - 1 + rnd) % (p - 1);
                const int i = min(a, b), j = max(a, b);
                pi[k] = i; pj[k] = j;
                const double aij = T[i * LD + j];
                double c = 1.0, sv = 0.0;
                if (aij != 0.0) {
                    const double tau = (T[j * LD + j] - T[i * LD + i]) / (2.0 * aij);
                    const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
                    c = 1.0 / sqrt(1.0 + t * t);
                    sv = t * c;
                }
                cs[k] = c; sn[k] = sv;
            }
            __syncthreads();
            // rows i, j of every pair (warp per pair, lanes along the row), then the columns
            for (int k = warp; k < half; k += nwarps) {
                const int i = pi[k], j = pj[k];
                const double c = cs[k], sv = sn[k];
                for (int l = lane; l < p; l += 32) {
                    const double ti = T[i * LD + l], tj = T[j * LD + l];
                    T[i * LD + l] = c * ti - sv * tj;
                    T[j * LD + l] = sv * ti + c * tj;
                }
            }
            __syncthreads();
            for (int k = warp; k < half; k += nwarps) {
                const int i = pi[k], j = pj[k];
                const double c = cs[k], sv = sn[k];
                for (int l = lane; l < p; l += 32) {
                    const double ti = T[l * LD + i], tj = T[l * LD + j];
                    T[l * LD + i] = c * ti - sv * tj;
                    T[l * LD + j] = sv * ti + c * tj;
                    const float qi = Q[l * LD + i], qj = Q[l * LD + j];
                    Q[l * LD + i] = (float)(c * qi - sv * qj);
                    Q[l * LD + j] = (float)(sv * qi + c * qj);
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < p; i += nt) {
        const double li = T[i * LD + i];
        int rank = 0;
        for (int j = 0; j < p; ++j) {
            const double lj = T[j * LD + j];
            rank += (lj > li) || (lj == li && j < i);
        }
        if (rank < r) {
            evals[rank] = li;
            for (int l = 0; l < p; ++l) Qsel[l * r + rank] = Q[l * LD + i];
        }
    }
}

inline size_t jacobi_smem(int p) {
    return (size_t)p * (p + 1) * sizeof(double) + (size_t)p * sizeof(double) +
           (size_t)p * (p + 1) * sizeof(float) + (size_t)p * sizeof(int);
}

// Columns of V (n x r): flip so that the largest-magnitude entry (first on ties) is positive.
__global__ void sign_fix_kernel(float *V, int n, int r) {
    const int c = blockIdx.x;
    __shared__ float bv[32];
    __shared__ int bi[32];
    float best = -1.f;
    int besti = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const float a = fabsf(V[(long long)i * r + c]);
        if (a > best) { best = a; besti = i; }
    }
    for (int o = 16; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o);
        const int oi = __shfl_xor_sync(0xffffffffu, besti, o);
        if (ob > best || (ob == best && oi < besti)) { best = ob; besti = oi; }
    }
    if ((threadIdx.x & 31) == 0) { bv[threadIdx.x >> 5] = best; bi[threadIdx.x >> 5] = besti; }
    __syncthreads();
    if (threadIdx.x == 0) {
        for (int w = 1; w < (int)(blockDim.x >> 5); ++w)
            if (bv[w] > best || (bv[w] == best && bi[w] < besti)) { best = bv[w]; besti = bi[w]; }
        bi[0] = besti;
    }
    __syncthreads();
    const bool flip = V[(long long)bi[0] * r + c] < 0.f;
    if (flip)
        for (int i = threadIdx.x; i < n; i += blockDim.x) V[(long long)i * r + c] = -V[(long long)i * r + c];
}

// l~ = lambda_rel * (sum diag H + sum diag C) / (n + r); then C += l~ I.
__global__ void il_lambda_kernel(const float *H, long long ldh, int n, double *C, int r,
                                 float lambda_rel, float *lam) {
    __shared__ double part[32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < n + r; i += blockDim.x) {
        const double d = i < n ? (double)H[(long long)i * ldh + i] : C[(i - n) * r + (i - n)];
        if (i < n && !isfinite(d)) report(GPTQ_ERR_NONFINITE, (long long)i * ldh + i);
        acc += d;
    }
    acc = warp_sum_d(acc);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
        v = warp_sum_d(v);
        if (threadIdx.x == 0) part[0] = v;
    }
    __syncthreads();
    const float l = (float)((double)lambda_rel * part[0] / (double)(n + r));
    if (threadIdx.x == 0) *lam = l;
    for (int i = threadIdx.x; i < r; i += blockDim.x) C[i * r + i] += (double)l;
}

struct ILWork {
    float *Y, *Z, *Qsel;       // subspace iteration blocks (n x p) and selected Ritz vectors
    double *HY, *Tm, *ev;      // fp64 Rayleigh-Ritz: H Y (n x p), Y^T H Y (p x p), values
    double *G, *Gi;            // p x p Gram and inverse UL factor
    double *B12, *Y1;          // n x r: H V and H V C^-1/2
    float *Yr;                 // n x r: H V C^-1
    double *C, *Ci;            // r x r extra block and inverse UL factor
    double *part;              // split-K partial sums of the fp64-accumulating products
    size_t part_elems;         // 4 n p
};

inline F64Split il_split(const ILWork &w) { return F64Split{w.part, w.part_elems}; }

constexpr int IL_ITERS_F32 = 4;   // power steps with fp32 accumulation
constexpr int IL_ITERS_F64 = 1;   // then with fp64 accumulation, before Rayleigh-Ritz

// dst = src Ubar^-T where src^T src = Ubar Ubar^T (Gram, factor and product in fp64):
// dst has orthonormal columns spanning src.
inline int cholqr_f64(const float *src, float *dst, int n, int p, ILWork &w, cudaStream_t s) {
    if (int st = gemm_f64acc<float, float, double>(p, p, n, src, p, 1, src, p, 0, w.G, p, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    if (int st = diag_ul_inv<double>(w.G, p, w.Gi, p, p, 0, s)) return st;
    return gemm_f64acc<float, double, float>(n, p, p, src, p, 0, w.Gi, p, 1, dst, p, 1.0,
            s, 0, F64Epilogue(), il_split(w));
}

// Top-r eigenvectors of H (n x n) into V (n x r).
inline int il_top_eigvecs(const float *H, long long ldh, int n, int r, float *V, ILWork &w,
                          cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_IL);
    const int p = il_block_p(n, r);
    random_block_kernel<<<256, 256, 0, s>>>(w.Y, (long long)n * p, 0x5eed0f11ull);
    GPTQ_CHECK_LAUNCH();
    for (int it = 0; it < IL_ITERS_F32 + IL_ITERS_F64; ++it) {
        // Z = H Y, then CholeskyQR2: Y <- orth(Z)
        if (it < IL_ITERS_F32) {
            if (int st = gemm_simt(gemm_args<float, float>(n, p, n, H, ldh, 0, w.Y, p, 0, w.Z, p, 1.f, 0.f), s)) return st;
        } else {
            if (int st = gemm_f64acc<float, float, float>(n, p, n, H, ldh, 0, w.Y, p, 0, w.Z, p, 1.0,
                    s, 0, F64Epilogue(), il_split(w))) return st;
        }
        if (int st = cholqr_f64(w.Z, w.Y, n, p, w, s)) return st;
        if (int st = cholqr_f64(w.Y, w.Z, n, p, w, s)) return st;
        std::swap(w.Y, w.Z);
    }
    // Rayleigh-Ritz in fp64: Tm = Y^T (H Y)
    if (int st = gemm_f64acc<float, float, double>(n, p, n, H, ldh, 0, w.Y, p, 0, w.HY, p, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    if (int st = gemm_f64acc<float, double, double>(p, p, n, w.Y, p, 1, w.HY, p, 0, w.Tm, p, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    const size_t smem = jacobi_smem(p);
    cudaFuncSetAttribute(jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    jacobi_eig_kernel<<<1, 512, smem, s>>>(w.Tm, p, r, w.Qsel, w.ev);
    GPTQ_CHECK_LAUNCH();
    // V = Y Qsel
    if (int st = gemm_f64acc<float, float, float>(n, r, p, w.Y, p, 0, w.Qsel, r, 0, V, r, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    sign_fix_kernel<<<r, 256, 0, s>>>(V, n, r);
    return launch_status();
}

// First n rows of U~ into Uaug (n x (n + r), ldu = n + r), lambda~ into *lam.
// The Schur complement S = H + l I - H V C^-1 V^T H cancels the large eigenvalues of H along
// V down to about l; it is formed with fp64 accumulation from the fp32 H and V, and only the
// (well conditioned) result is rounded to fp32 for the factor.
// Awork: n x n scratch, T: FACTOR_NB x n scratch.
inline int il_factor(const float *H, long long ldh, int n, int r, const float *V,
                     float lambda_rel, float *Uaug, float *Awork, float *T, float *lam,
                     ILWork &w, cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_IL);
    const long long ldu = n + r;
    // B12 = H V (n x r), C = V^T B12 (r x r)
    if (int st = gemm_f64acc<float, float, double>(n, r, n, H, ldh, 0, V, r, 0, w.B12, r, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    if (int st = gemm_f64acc<float, double, double>(r, r, n, V, r, 1, w.B12, r, 0, w.C, r, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    il_lambda_kernel<<<1, 1024, 0, s>>>(H, ldh, n, w.C, r, lambda_rel, lam);
    GPTQ_CHECK_LAUNCH();
    // C = Ubar Ubar^T, Ci = Ubar^-1, C^-1 = Ci^T Ci
    if (int st = diag_ul_inv<double>(w.C, r, w.Ci, r, r, 0, s)) return st;
    // Y1 = B12 Ci^T, Yr = Y1 Ci = B12 C^-1
    if (int st = gemm_f64acc<double, double, double>(n, r, r, w.B12, r, 0, w.Ci, r, 1, w.Y1, r, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    if (int st = gemm_f64acc<double, double, float>(n, r, r, w.Y1, r, 0, w.Ci, r, 0, w.Yr, r, 1.0,
            s, 1, F64Epilogue(), il_split(w))) return st;
    // S = H + l I - Y1 Y1^T (upper triangle), fp64 accumulation, fp32 result
    F64Epilogue ep;
    ep.Cin = H; ep.ldcin = ldh; ep.beta = 1.0; ep.diag = lam; ep.c_upper = 1;
    if (int st = gemm_f64acc<double, double, float>(n, n, r, w.Y1, r, 0, w.Y1, r, 1, Awork, n, -1.0,
            s, 0, ep, il_split(w))) return st;
    cudaMemsetAsync(Uaug, 0, sizeof(float) * (size_t)n * ldu, s);
    if (int st = factor_ul_inverse(Awork, n, Uaug, ldu, n, T, s)) return st;
    // U12 = -U11 Yr
    auto p = gemm_args<float, float>(n, r, n, Uaug, ldu, 0, w.Yr, r, 0, Uaug + n, ldu, -1.f, 0.f);
    p.a_upper = 1;
    return gemm_f32(p, s);
}

}  // namespace gptq
