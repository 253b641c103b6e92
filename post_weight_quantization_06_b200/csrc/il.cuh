// GPTQ-intrinsic LoRA on the device.
//
// GPTQ-intrinsic LoRA summary, "Method" part 2: X~ = [X, X V_r] with V_r the top-r right
// singular vectors of X; the pass runs on W~ = [W, 0]; the r extra coordinates absorb the
// error and become R; the singular augmented Hessian is factored without a plain Cholesky.
//
// Device route:
//   1. V_r: block subspace iteration on H (= 2 X^T X, same eigenvectors as X^T X): a few
//      fp32-accurate tensor-core power steps, then fp64 iterations with CholeskyQR2
//      re-orthonormalisation and a Rayleigh-Ritz step (eig.cuh) until every top-r Ritz pair
//      passes a relative residual test (see il_top_eigvecs).
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
#include "eig.cuh"

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

// Columns of V64 (n x r, fp64): flip so that the largest-magnitude entry (first on ties) is
// positive; the same flip goes to the matching column of Qr (p x r), and V (fp32) receives the
// rounded result.
__global__ void sign_fix_kernel(double *V64, float *V, int n, int r, double *Qr, int p) {
    const int c = blockIdx.x;
    __shared__ double bv[32];
    __shared__ int bi[32];
    double best = -1.0;
    int besti = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const double a = fabs(V64[(long long)i * r + c]);
        if (a > best) { best = a; besti = i; }
    }
    for (int o = 16; o > 0; o >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, o);
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
    const double sg = V64[(long long)bi[0] * r + c] < 0.0 ? -1.0 : 1.0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const double v = sg * V64[(long long)i * r + c];
        V64[(long long)i * r + c] = v;
        V[(long long)i * r + c] = (float)v;
    }
    for (int k = threadIdx.x; k < p; k += blockDim.x) Qr[(long long)k * r + c] *= sg;
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

// Control words of the eigenvector iteration (device memory, see il_top_eigvecs): per phase a
// done flag and a count of residual tests, and the residual kernel's CTA counter.
enum {
    IL_CTL_DONE = 0, IL_CTL_ITERS = 1,     // phase 2 (fp64)
    IL_CTL_DONE1 = 2, IL_CTL_CHECKS1 = 3,  // phase 1 (fp32-accurate tensor-core products)
    IL_CTL_COUNTER = 4, IL_CTL_WORDS = 8
};

// Relative residuals of the top r Ritz pairs, r_c = || H v_c - theta_c v_c || / theta_c with
// v_c = Y Qr[:, c] and H v_c = HY Qr[:, c] (fp64 arithmetic). Each CTA sums r_c^2 over 32 rows
// for 64 columns and writes its partial; the last CTA to finish adds the partials in a fixed
// order and takes the decision of its phase:
//   phase 2: done when max_c r_c <= tol;
//   phase 1: done when max_c r_c <= tol or when it is above half the previous test's value
//            (the fp32-accurate products have reached their floor);
// it counts the test and stores max_c r_c in *resid. Nothing happens once the phase is done.
constexpr int RES_ROWS = 32, RES_COLS = 64, RES_THREADS = 256;

inline size_t il_residual_smem(int p) {
    return sizeof(double) * ((size_t)p * RES_COLS + 2 * (size_t)RES_ROWS * p);
}

template <typename THY>
__global__ __launch_bounds__(RES_THREADS) void il_residual_kernel(
    const THY *HY, const float *Y, const double *Qr, const double *ev, int n, int p, int r,
    double *part, int *ctl, int phase, double tol, double *resid) {
    const int done_w = phase == 1 ? IL_CTL_DONE1 : IL_CTL_DONE;
    const int count_w = phase == 1 ? IL_CTL_CHECKS1 : IL_CTL_ITERS;
    pdl_wait_prev();
    pdl_launch_next();
    if (ctl[done_w]) return;
    extern __shared__ __align__(16) double rsm[];
    double *Qc = rsm;                        // p x 64
    double *HYs = Qc + p * RES_COLS;         // 32 x p
    double *Ys = HYs + RES_ROWS * p;         // 32 x p
    __shared__ double red[RES_THREADS / RES_COLS][RES_COLS];
    __shared__ int last;
    const int tid = threadIdx.x;
    const int c0 = blockIdx.y * RES_COLS, i0 = blockIdx.x * RES_ROWS;
    const int nc = min(RES_COLS, r - c0);
    for (int idx = tid; idx < p * RES_COLS; idx += RES_THREADS) {
        const int k = idx / RES_COLS, c = idx % RES_COLS;
        Qc[idx] = c < nc ? Qr[(long long)k * r + c0 + c] : 0.0;
    }
    for (int idx = tid; idx < RES_ROWS * p; idx += RES_THREADS) {
        const int i = idx / p, k = idx % p;
        const long long row = i0 + i;
        HYs[idx] = row < n ? (double)HY[row * p + k] : 0.0;
        Ys[idx] = row < n ? (double)Y[row * p + k] : 0.0;
    }
    __syncthreads();
    const int c = tid % RES_COLS, g = tid / RES_COLS;
    const double th = c < nc ? ev[c0 + c] : 0.0;
    double acc = 0.0;
    for (int i = g; i < RES_ROWS; i += RES_THREADS / RES_COLS) {
        double a = 0.0, b = 0.0;
        for (int k = 0; k < p; ++k) {
            const double q = Qc[k * RES_COLS + c];
            a = fma(HYs[i * p + k], q, a);
            b = fma(Ys[i * p + k], q, b);
        }
        const double rr = fma(-th, b, a);
        acc = fma(rr, rr, acc);
    }
    red[g][c] = acc;
    __syncthreads();
    const int nblk = gridDim.x;
    if (tid < nc) {
        double t = 0.0;
        for (int gg = 0; gg < RES_THREADS / RES_COLS; ++gg) t += red[gg][tid];
        part[(long long)(c0 + tid) * nblk + blockIdx.x] = t;
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) last = atomicAdd(&ctl[IL_CTL_COUNTER], 1) == (int)(gridDim.x * gridDim.y) - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    double worst = 0.0;
    const double floor = 1e-300 + 1e-14 * fabs(ev[0]);
    for (int cc = tid; cc < r; cc += RES_THREADS) {
        double t = 0.0;
        for (int b = 0; b < nblk; ++b) t += *((volatile double *)&part[(long long)cc * nblk + b]);
        worst = fmax(worst, sqrt(t) / fmax(fabs(ev[cc]), floor));
    }
    for (int o = 16; o > 0; o >>= 1) worst = fmax(worst, __shfl_xor_sync(0xffffffffu, worst, o));
    __shared__ double wmax[RES_THREADS / 32];
    if ((tid & 31) == 0) wmax[tid >> 5] = worst;
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < RES_THREADS / 32; ++w) worst = fmax(worst, wmax[w]);
        const double prev = *resid;
        const bool stalled = phase == 1 && ctl[count_w] > 0 && worst > 0.5 * prev;
        *resid = worst;
        ctl[count_w] += 1;
        ctl[IL_CTL_COUNTER] = 0;
        ctl[done_w] = (worst <= tol || stalled) ? 1 : 0;
    }
}

// After the capped loop: GPTQ_ERR_NOT_CONVERGED (info = iterations run) if the residual test
// never passed.
__global__ void il_finish_kernel(const int *ctl) {
    if (threadIdx.x == 0 && !ctl[IL_CTL_DONE]) report(GPTQ_ERR_NOT_CONVERGED, ctl[IL_CTL_ITERS]);
}

struct ILWork {
    float *Y, *Z;              // n x p subspace blocks (fp32)
    double *HY;                // n x p: H Y (fp64)
    double *Tm, *ev, *Qr;      // Rayleigh-Ritz: Y^T H Y (p x p), Ritz values (p), vectors (p x r)
    double *G, *Gi;            // p x p Gram and inverse UL factor (orthonormalisation)
    double *V64;               // n x r Ritz vectors Y Qr
    double *B12, *Y1;          // n x r: H V and H V C^-1/2
    float *Yr;                 // n x r: H V C^-1
    double *C, *Ci;            // r x r extra block and inverse UL factor
    double *res;               // residual partials (r x row blocks) and the last residual
    int *ctl;                  // IL_CTL_WORDS control words
    double *part;              // split-K partial sums of the fp64-accumulating products
    size_t part_elems;         // 4 n p
};

inline F64Split il_split(const ILWork &w) { return F64Split{w.part, w.part_elems}; }

inline F64Epilogue skip_if(const int *flag) {
    F64Epilogue ep;
    ep.skip = flag;
    return ep;
}

// Stopping rule of the eigenvector iteration: every one of the top r Ritz pairs has
// || H v - theta v || <= IL_TOL * theta, with at most IL_MAX_ITERS fp64 iterations
// (GPTQ_IL_MAX_ITERS overrides the cap, read at each call). Phase 1 runs at most
// IL_P1_STEPS power steps with a residual test every IL_P1_EVERY steps.
constexpr int IL_P1_STEPS = 24, IL_P1_EVERY = 4;
constexpr double IL_P1_TOL = 1e-4;
constexpr int IL_MAX_ITERS = 12;
constexpr double IL_TOL = 5e-6;

// dst = src Ubar^-T where src^T src = Ubar Ubar^T (Gram, factor and product in fp64):
// dst has orthonormal columns spanning src.
template <typename TS>
inline int cholqr_f64(const TS *src, float *dst, int n, int p, ILWork &w, cudaStream_t s,
                      const int *skip = nullptr) {
    if (int st = gemm_f64acc<TS, TS, double>(p, p, n, src, p, 1, src, p, 0, w.G, p, 1.0,
            s, 0, skip_if(skip), il_split(w))) return st;
    if (int st = diag_ul_inv<double>(w.G, p, w.Gi, p, p, 0, s, skip)) return st;
    return gemm_f64acc<TS, double, float>(n, p, p, src, p, 0, w.Gi, p, 1, dst, p, 1.0,
            s, 0, skip_if(skip), il_split(w));
}

// Top-r eigenvectors of the symmetric n x n matrix H: V (n x r, fp32, decreasing eigenvalue,
// largest-magnitude entry of each column positive); also V64 (fp64) and B12 = H V64 in the
// workspace. Subspace iteration on a block of p columns:
//   phase 1: power steps Y <- orth(H Y) with fp32-accurate tensor-core products, until a
//            residual test every IL_P1_EVERY steps passes IL_P1_TOL or stops improving;
//   phase 2: up to the cap, each iteration (after the first) Y <- orth(HY) twice over
//            (CholeskyQR2), then HY = H Y and T = Y^T HY with fp64 accumulation, the top r
//            eigenpairs of T (sym_eig_top), and the residual test. Once it passes, a device
//            flag makes every later launch of the loop return at once, so Y, HY and the
//            Ritz pairs stay those of the converged iteration.
inline int il_top_eigvecs(const float *H, long long ldh, int n, int r, float *V, ILWork &w,
                          cudaStream_t s, bool want_b12 = true) {
    KtStageScope stage(GPTQ_KT_IL);
    const int p = il_block_p(n, r);
    static const long long cap_env = tc::env_ll("GPTQ_IL_MAX_ITERS", 0);
    const long long cap_now = tc::env_ll("GPTQ_IL_MAX_ITERS", cap_env);
    const int cap = cap_now > 0 ? (int)std::min<long long>(cap_now, 64) : IL_MAX_ITERS;
    const int *done = w.ctl + IL_CTL_DONE, *done1 = w.ctl + IL_CTL_DONE1;
    if (cudaMemsetAsync(w.ctl, 0, sizeof(int) * IL_CTL_WORDS, s) != cudaSuccess) return GPTQ_ERR_CUDA;
    random_block_kernel<<<256, 256, 0, s>>>(w.Y, (long long)n * p, 0x5eed0f11ull);
    GPTQ_CHECK_LAUNCH();
    const int nblk = ceil_div(n, RES_ROWS);
    const dim3 rgrid(nblk, ceil_div(r, RES_COLS));
    const size_t rsmem = il_residual_smem(p);
    double *resid = w.res + (size_t)r * nblk;
    GPTQ_SMEM_LIMIT(il_residual_kernel<float>, il_residual_smem(EIG_MAXP));
    GPTQ_SMEM_LIMIT(il_residual_kernel<double>, il_residual_smem(EIG_MAXP));
    // phase 1: Z = H Y on the tensor cores (fp32 accuracy), Y = orth(Z); every IL_P1_EVERY
    // steps the Ritz pairs of Y (from Z) are tested first
    for (int it = 0; it < IL_P1_STEPS; ++it) {
        auto pz = gemm_args<float, float>(n, p, n, H, ldh, 0, w.Y, p, 0, w.Z, p, 1.f, 0.f);
        pz.skip = done1;
        pz.pdl = 1;
        if (int st = gemm_f32(pz, s)) return st;
        if (it > 0 && it % IL_P1_EVERY == 0) {
            if (int st = gemm_f64acc<float, float, double>(p, p, n, w.Y, p, 1, w.Z, p, 0, w.Tm, p,
                    1.0, s, 0, skip_if(done1), il_split(w))) return st;
            if (int st = sym_eig_top(w.Tm, p, r, w.ev, w.Qr, done1, s)) return st;
            if (int st = launch_kernel(il_residual_kernel<float>, rgrid, dim3(RES_THREADS), rsmem, s,
                                       true, (const float *)w.Z, (const float *)w.Y,
                                       (const double *)w.Qr, (const double *)w.ev, n, p, r, w.res,
                                       w.ctl, 1, IL_P1_TOL, resid))
                return st;
        }
        if (int st = cholqr_f64<float>(w.Z, w.Y, n, p, w, s, done1)) return st;
    }
    // phase 2: fp64 products, a residual test every iteration
    for (int it = 0; it < cap; ++it) {
        if (it > 0) {
            if (int st = cholqr_f64<double>(w.HY, w.Z, n, p, w, s, done)) return st;
            if (int st = cholqr_f64<float>(w.Z, w.Y, n, p, w, s, done)) return st;
        }
        if (int st = gemm_f64acc<float, float, double>(n, p, n, H, ldh, 0, w.Y, p, 0, w.HY, p,
                1.0, s, 0, skip_if(done), il_split(w))) return st;
        if (int st = gemm_f64acc<float, double, double>(p, p, n, w.Y, p, 1, w.HY, p, 0, w.Tm, p,
                1.0, s, 0, skip_if(done), il_split(w))) return st;
        if (int st = sym_eig_top(w.Tm, p, r, w.ev, w.Qr, done, s)) return st;
        if (int st = launch_kernel(il_residual_kernel<double>, rgrid, dim3(RES_THREADS), rsmem, s,
                                   true, (const double *)w.HY, (const float *)w.Y,
                                   (const double *)w.Qr, (const double *)w.ev, n, p, r, w.res,
                                   w.ctl, 2, IL_TOL, resid))
            return st;
    }
    il_finish_kernel<<<1, 32, 0, s>>>(w.ctl);
    GPTQ_CHECK_LAUNCH();
    // V64 = Y Qr, signs fixed (Qr's columns follow), V = fp32(V64); B12 = H V64 = HY Qr
    if (int st = gemm_f64acc<float, double, double>(n, r, p, w.Y, p, 0, w.Qr, r, 0, w.V64, r, 1.0,
            s, 0, F64Epilogue(), il_split(w))) return st;
    sign_fix_kernel<<<r, 256, 0, s>>>(w.V64, V, n, r, w.Qr, p);
    GPTQ_CHECK_LAUNCH();
    if (!want_b12) return GPTQ_OK;
    return gemm_f64acc<double, double, double>(n, r, p, w.HY, p, 0, w.Qr, r, 0, w.B12, r, 1.0,
            s, 0, F64Epilogue(), il_split(w));
}

// First n rows of U~ into Uaug (n x (n + r), ldu = n + r), lambda~ into *lam, from the
// eigenvector step's V64 and B12 = H V64 (both fp64; V, the fp32 output, is V64 rounded).
// The Schur complement S = H + l I - H V C^-1 V^T H cancels the large eigenvalues of H along
// V down to about l; it is formed with fp64 accumulation from the fp32 H, and only the (well
// conditioned) result is rounded to fp32 for the factor.
// Awork: n x n scratch, T: FACTOR_NB x n scratch.
inline int il_factor(const float *H, long long ldh, int n, int r, float lambda_rel, float *Uaug,
                     float *Awork, float *T, float *lam, ILWork &w, cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_IL);
    const long long ldu = n + r;
    // C = V64^T B12 (r x r)
    if (int st = gemm_f64acc<double, double, double>(r, r, n, w.V64, r, 1, w.B12, r, 0, w.C, r,
            1.0, s, 0, F64Epilogue(), il_split(w))) return st;
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
    if (cudaMemsetAsync(Uaug, 0, sizeof(float) * (size_t)n * ldu, s) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    if (int st = factor_ul_inverse(Awork, n, Uaug, ldu, n, T, s)) return st;
    // U12 = -U11 Yr
    auto pa = gemm_args<float, float>(n, r, n, Uaug, ldu, 0, w.Yr, r, 0, Uaug + n, ldu, -1.f, 0.f);
    pa.a_upper = 1;
    return gemm_f32(pa, s);
}

}  // namespace gptq
