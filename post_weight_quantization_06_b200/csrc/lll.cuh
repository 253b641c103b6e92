// GPTQ with lattice basis reduction (WITHREDUCTION) on the device.
//
// The Lattice Geometry of Neural Network Quantization, section 5.2 ("Use of lattice basis
// reduction"): reduce the basis of the regularised data lattice X' = [X; mu I] with LLL before
// running GPTQ / Babai on it; the coefficients found in the reduced basis map back through the
// unimodular change of basis T, and large entries of T can push codes out of range.
//
// With one scale per output row (per-channel grid) every row's lattice is s X', so one
// reduction of X' (Gram matrix G' = X'^T X' = (H + lambda I) / 2) serves the whole layer:
//   1. lambda = lambda_rel mean(diag H); G' in fp64, its columns reversed (GPTQ visits the
//      columns in natural order, which is Babai's nearest plane on the reversed basis);
//   2. LLL (Lenstra, Lenstra and Lovasz 1982; delta = 3/4) on the Gram matrix, one CTA in
//      fp64: the Gram-Schmidt data from a Cholesky factor, then size reductions and swaps with
//      the classical updates of mu and the squared Gram-Schmidt lengths, T and T^-1 kept
//      alongside (rows of T^-1 receive the inverse elementary operations);
//   3. per row the min-max grid (s, z) and its coordinates u = w / s + z; u' = T^-1 u;
//   4. one-sided adaptive rounding of u' under G_red = T^T G' T (the two-sided wavefront with
//      the left Gram matrix the identity): Babai's nearest plane in the reduced basis;
//   5. c = clip(T c', 0, maxq), counted where clipping changed a code; packed codes and the
//      loss (w - w_hat)^T (H + lambda I) (w - w_hat).
#pragma once

#include "common.cuh"

namespace gptq {

constexpr int LLL_THREADS = 1024;
constexpr int LLL_MAX_N = 2048;

// A[i][j] = G'[n-1-i][n-1-j] in fp64 (reversed order) and Gd = G' in fp32 (natural order), with
// G' = (H_sym + lambda I) / 2, H_sym read from H's upper triangle.
__global__ void lll_prep_kernel(const float *H, long long ldh, int n, const float *lam, double *A,
                                float *Gd) {
    const double l = (double)*lam;
    const long long total = (long long)n * n;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(idx / n), j = (int)(idx % n);
        const int a = min(i, j), b = max(i, j);
        const double g = 0.5 * ((double)H[(long long)a * ldh + b] + (i == j ? l : 0.0));
        Gd[idx] = (float)g;
        A[(long long)(n - 1 - i) * n + (n - 1 - j)] = g;
    }
}

// One CTA. A: n x n fp64 Gram matrix of the (reversed) basis, overwritten (its lower triangle
// ends as the Gram-Schmidt coefficients mu). Bn: n squared Gram-Schmidt lengths. T, Ti: n x n
// fp64, written with the unimodular T (reduced basis = B T) and T^-1. stats: [swaps, size
// reductions, loop iterations]. The arithmetic of the updates is written out with
// round-to-nearest operations (no contraction into FMAs), in the order of the textbook
// formulas. A bounded loop: past max_iter iterations it stops and reports
// GPTQ_ERR_NOT_CONVERGED (info = swaps).
__global__ __launch_bounds__(LLL_THREADS) void lll_kernel(double *A, int n, double *Bn, double *T,
                                                          double *Ti, long long *stats,
                                                          long long max_iter, double delta) {
    __shared__ double sd;
    __shared__ int sl;
    __shared__ double colj[LLL_MAX_N];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = LLL_THREADS / 32;
    auto at = [&](int i, int j) -> double & { return A[(long long)i * n + j]; };
    // ---- Cholesky G = L L^T (lower, right-looking)
    for (int j = 0; j < n; ++j) {
        if (tid == 0) {
            double d = at(j, j);
            if (!(d > 0.0) || !isfinite(d)) {
                report(GPTQ_ERR_NOT_PD, j);
                d = 1e-300;
            }
            sd = sqrt(d);
            at(j, j) = sd;
        }
        __syncthreads();
        const double ljj = sd;
        for (int i = j + 1 + tid; i < n; i += LLL_THREADS) {
            const double v = at(i, j) / ljj;
            at(i, j) = v;
            colj[i] = v;
        }
        __syncthreads();
        for (int i = j + 1 + warp; i < n; i += NW) {
            const double aij = colj[i];
            for (int k = j + 1 + lane; k <= i; k += 32) at(i, k) -= aij * colj[k];
        }
        __syncthreads();
    }
    // ---- mu[i][j] = L[i][j] / L[j][j] (strictly lower), Bn[i] = L[i][i]^2
    for (int i = tid; i < n; i += LLL_THREADS) Bn[i] = at(i, i) * at(i, i);
    for (long long idx = tid; idx < (long long)n * n; idx += LLL_THREADS) {
        const int i = (int)(idx / n), j = (int)(idx % n);
        if (j < i) at(i, j) = at(i, j) / at(j, j);
        T[idx] = i == j ? 1.0 : 0.0;
        Ti[idx] = i == j ? 1.0 : 0.0;
    }
    __syncthreads();
    long long swaps = 0, reds = 0, it = 0;
    // b_k <- b_k - q b_l with q = rint(mu[k][l]) (nothing when q == 0)
    auto reduce = [&](int k, int l) {
        const double q = rint(at(k, l));
        __syncthreads();
        if (q != 0.0) {
            for (int j = tid; j < l; j += LLL_THREADS) at(k, j) = __dsub_rn(at(k, j), __dmul_rn(q, at(l, j)));
            if (tid == 0) at(k, l) = __dsub_rn(at(k, l), q);
            for (int i = tid; i < n; i += LLL_THREADS) {
                T[(long long)i * n + k] -= q * T[(long long)i * n + l];
                Ti[(long long)l * n + i] += q * Ti[(long long)k * n + i];
            }
            ++reds;
        }
        __syncthreads();
    };
    int k = 1;
    while (k < n) {
        if (++it > max_iter) {
            if (tid == 0) report(GPTQ_ERR_NOT_CONVERGED, swaps);
            break;
        }
        reduce(k, k - 1);
        const double m = at(k, k - 1);
        const double bk = Bn[k], bk1 = Bn[k - 1];
        __syncthreads();
        if (bk < __dmul_rn(__dsub_rn(delta, __dmul_rn(m, m)), bk1)) {
            // swap b_{k-1} and b_k
            const double B = __dadd_rn(bk, __dmul_rn(__dmul_rn(m, m), bk1));
            const double mnew = __ddiv_rn(__dmul_rn(m, bk1), B);
            for (int j = tid; j < k - 1; j += LLL_THREADS) {
                const double t = at(k - 1, j);
                at(k - 1, j) = at(k, j);
                at(k, j) = t;
            }
            for (int i = tid; i < n; i += LLL_THREADS) {
                double t = T[(long long)i * n + k - 1];
                T[(long long)i * n + k - 1] = T[(long long)i * n + k];
                T[(long long)i * n + k] = t;
                t = Ti[(long long)(k - 1) * n + i];
                Ti[(long long)(k - 1) * n + i] = Ti[(long long)k * n + i];
                Ti[(long long)k * n + i] = t;
            }
            for (int i = k + 1 + tid; i < n; i += LLL_THREADS) {
                const double t = at(i, k);
                const double nk = __dsub_rn(at(i, k - 1), __dmul_rn(m, t));
                at(i, k) = nk;
                at(i, k - 1) = __dadd_rn(t, __dmul_rn(mnew, nk));
            }
            __syncthreads();
            if (tid == 0) {
                at(k, k - 1) = mnew;
                Bn[k] = __ddiv_rn(__dmul_rn(bk1, bk), B);
                Bn[k - 1] = B;
            }
            __syncthreads();
            ++swaps;
            k = k > 1 ? k - 1 : 1;
        } else {
            // size reduction against l = k-2 .. 0: the next l with |mu[k][l]| > 1/2 (the only
            // ones with q != 0) is found by a scan of the whole row
            int l = k - 2;
            while (l >= 0) {
                if (tid == 0) sl = -1;
                __syncthreads();
                int best = -1;
                for (int j = tid; j <= l; j += LLL_THREADS)
                    if (fabs(at(k, j)) > 0.5) best = j;
                for (int o = 16; o > 0; o >>= 1) best = max(best, __shfl_xor_sync(0xffffffffu, best, o));
                if (lane == 0 && best >= 0) atomicMax(&sl, best);
                __syncthreads();
                const int ls = sl;
                __syncthreads();
                if (ls < 0) break;
                reduce(k, ls);
                l = ls - 1;
            }
            ++k;
        }
    }
    if (tid == 0) {
        stats[0] = swaps;
        stats[1] = reds;
        stats[2] = it;
    }
}

// T and T^-1 back in GPTQ's column order (Tf[i][j] = T[n-1-i][n-1-j]) as fp32; entries beyond
// 2^24 (not exact in fp32) report GPTQ_ERR_NOT_CONVERGED (info -1). stats[3] = max |T|.
__global__ void lll_export_kernel(const double *T, const double *Ti, int n, float *Tf, float *Tif,
                                  long long *stats) {
    double mx = 0.0;
    const long long total = (long long)n * n;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(idx / n), j = (int)(idx % n);
        const long long src = (long long)(n - 1 - i) * n + (n - 1 - j);
        const double t = T[src], u = Ti[src];
        mx = fmax(mx, fmax(fabs(t), fabs(u)));
        Tf[idx] = (float)t;
        Tif[idx] = (float)u;
    }
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if ((threadIdx.x & 31) == 0) {
        if (mx > 16777216.0) report(GPTQ_ERR_NOT_CONVERGED, -1);
        atomicMax(reinterpret_cast<unsigned long long *>(stats + 3), (unsigned long long)mx);
    }
}

// Per row: the min-max grid over the whole row (one group), s and z written to scales / zeros,
// and the row's grid coordinates U = W / s + z. One warp per row.
template <typename TW>
__global__ void rowgrid_kernel(const TW *W, int m, int n, int bits, float *scales, uint8_t *zeros,
                               float *U) {
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (row >= m) return;
    const TW *w = W + (long long)row * n;
    float mn = INFINITY, mx = -INFINITY;
    for (int j = lane; j < n; j += 32) {
        const float v = to_f32(w[j]);
        if (!isfinite(v)) report(GPTQ_ERR_NONFINITE, (long long)row * n + j);
        mn = fminf(mn, v);
        mx = fmaxf(mx, v);
    }
    mn = warp_min(mn);
    mx = warp_max(mx);
    const float fmaxq = (float)((1 << bits) - 1);
    mn = fminf(mn, 0.f);
    mx = fmaxf(mx, 0.f);
    if (mx == mn) { mn = -1.f; mx = 1.f; }
    const float s = __fdiv_rn(mx - mn, fmaxq);
    const float z = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.f), fmaxq);
    if (lane == 0) {
        scales[row] = s;
        zeros[row] = (uint8_t)z;
    }
    for (int j = lane; j < n; j += 32) U[(long long)row * n + j] = __fdiv_rn(to_f32(w[j]), s) + z;
}

__global__ void int_to_float_kernel(const int32_t *Z, long long total, float *F) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x)
        F[i] = (float)Z[i];
}

// Codes c = clip(rint(Cr), 0, maxq) (Cr = T c' holds integers), one byte each; D = W - s (c - z)
// for the loss; stats[4] += the number of codes that clipping changed.
template <typename TW>
__global__ void reduced_codes_kernel(const float *Cr, const TW *W, const float *scales,
                                     const uint8_t *zeros, int m, int n, int bits, uint8_t *c8,
                                     float *D, long long *stats) {
    const float fmaxq = (float)((1 << bits) - 1);
    const long long total = (long long)m * n;
    unsigned long long clipped = 0;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int row = (int)(idx / n);
        const float raw = rintf(Cr[idx]);
        const float c = fminf(fmaxf(raw, 0.f), fmaxq);
        clipped += c != raw;
        c8[idx] = (uint8_t)c;
        D[idx] = to_f32(W[idx]) - scales[row] * (c - (float)zeros[row]);
    }
    for (int o = 16; o > 0; o >>= 1) clipped += __shfl_xor_sync(0xffffffffu, clipped, o);
    if ((threadIdx.x & 31) == 0 && clipped)
        atomicAdd(reinterpret_cast<unsigned long long *>(stats + 4), clipped);
}

// Packs one byte per code into the LSB-first bit stream of 32-bit words (row stride n*bits/32).
__global__ void pack_codes_kernel(const uint8_t *c8, int m, int n, int bits, uint32_t *codes) {
    const long long words = (long long)n * bits / 32;
    const long long total = (long long)m * words;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long row = idx / words, wd = idx % words;
        const long long bit0 = wd * 32;
        const long long cfirst = bit0 / bits, clast = min((long long)n - 1, (bit0 + 31) / bits);
        uint32_t word = 0;
        for (long long c = cfirst; c <= clast; ++c) {
            const long long pos = c * bits - bit0;
            const uint32_t code = c8[row * n + c];
            word |= pos >= 0 ? (code << pos) : (code >> (-pos));
        }
        codes[idx] = word;
    }
}

}  // namespace gptq
