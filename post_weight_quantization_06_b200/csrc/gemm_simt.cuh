// Generic fp32-accumulating SIMT GEMM: C = alpha * op(A) op(B) + beta * C, with optional
// triangular structure. Used where a step is a small or awkward contraction (panel solves,
// the fp32-input Hessian); large contractions go to the tcgen05 kernels.
#pragma once

#include "common.cuh"
#include "ktimes.cuh"

namespace gptq {

template <typename TA, typename TB>
struct GemmArgs {
    int M, N, K;
    const TA *A;
    long long lda;
    int ta;  // A(i,k) = ta ? A[k*lda + i] : A[i*lda + k]
    const TB *B;
    long long ldb;
    int tb;  // B(k,j) = tb ? B[j*ldb + k] : B[k*ldb + j]
    float *C;
    long long ldc;
    float alpha, beta;  // beta == 0: C is not read
    int c_upper;        // write only C(i,j) with j >= i (tiles strictly below are skipped)
    int a_upper;        // A(i,k) = 0 for k < i (storage there is not read)
    int b_upper;        // B(k,j) = 0 for k > j (storage there is not read)
    int a_lower;        // A(i,k) = 0 for k > i
    int b_lower;        // B(k,j) = 0 for k < j
    int max_ctas;       // > 0: at most this many persistent CTAs (tensor-core path only), so
                        // that kernels on other streams keep SMs
    int pdl;            // launch as a programmatic dependent of the stream's previous kernel
                        // (the launch and the setup overlap that kernel's tail)
    const int *skip;    // when set and *skip != 0 the launch does nothing
    const float *a_lo;  // A given as tf32 hi (A) and lo (a_lo, same layout): op(A) = A + a_lo
    const float *b_lo;  // B likewise: op(B) = B + b_lo (tensor-core and fp32 paths only)
    const float *b_full;  // with b_lo: the unsplit B (row stride ldb_full), which the SIMT
    long long ldb_full;   // path takes instead of the two parts
};

namespace simt {
constexpr int NT = 256;
}

// BT x BT output tile per CTA of 256 threads (16 x 16), each thread a TM x TM sub-tile made
// of TM/4 x TM/4 float4 blocks BT/2 apart; BT = 128 for large products, 64 for small ones
// (four times as many CTAs, a K slice of 32).
template <typename TA, typename TB, int BT>
__global__ __launch_bounds__(256) void gemm_simt_kernel(GemmArgs<TA, TB> p) {
    using namespace simt;
    constexpr int BM = BT, BN = BT, BK = 2048 / BT, TM = BT / 16, NH = TM / 4;
    const int i0 = blockIdx.y * BM, j0 = blockIdx.x * BN;
    if (p.c_upper && i0 >= j0 + BN) return;
    pdl_wait_prev();
    if (p.skip && *p.skip) return;
    __shared__ __align__(16) float As[BK][BM + 4];
    __shared__ __align__(16) float Bs[BK][BN + 4];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    float acc[TM][TM];
#pragma unroll
    for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TM; ++j) acc[i][j] = 0.f;

    int kbeg = 0, kend = p.K;
    if (p.a_upper) kbeg = max(kbeg, i0);
    if (p.b_upper) kend = min(kend, j0 + BN);
    if (p.a_lower) kend = min(kend, i0 + BM);
    if (p.b_lower) kbeg = max(kbeg, j0);
    kbeg = (kbeg / BK) * BK;

    // register double buffering: the global loads of K tile k+1 are in flight while tile k
    // is multiplied out of shared memory
    float ra[(BM * BK) / NT], rb[(BN * BK) / NT];
    auto load_tiles = [&](int k0) {
#pragma unroll
        for (int e = 0; e < (BM * BK) / NT; ++e) {
            const int idx = tid + e * NT;
            int r, kk;
            if (p.ta) { kk = idx / BM; r = idx % BM; } else { r = idx / BK; kk = idx % BK; }
            const int gi = i0 + r, gk = k0 + kk;
            float v = 0.f;
            if (gi < p.M && gk < kend && (!p.a_upper || gk >= gi) && (!p.a_lower || gk <= gi))
                v = to_f32(p.ta ? p.A[(long long)gk * p.lda + gi] : p.A[(long long)gi * p.lda + gk]);
            ra[e] = v;
        }
#pragma unroll
        for (int e = 0; e < (BN * BK) / NT; ++e) {
            const int idx = tid + e * NT;
            int c, kk;
            if (p.tb) { c = idx / BK; kk = idx % BK; } else { kk = idx / BN; c = idx % BN; }
            const int gj = j0 + c, gk = k0 + kk;
            float v = 0.f;
            if (gj < p.N && gk < kend && (!p.b_upper || gk <= gj) && (!p.b_lower || gk >= gj))
                v = to_f32(p.tb ? p.B[(long long)gj * p.ldb + gk] : p.B[(long long)gk * p.ldb + gj]);
            rb[e] = v;
        }
    };
    if (kbeg < kend) load_tiles(kbeg);
    for (int k0 = kbeg; k0 < kend; k0 += BK) {
#pragma unroll
        for (int e = 0; e < (BM * BK) / NT; ++e) {
            const int idx = tid + e * NT;
            int r, kk;
            if (p.ta) { kk = idx / BM; r = idx % BM; } else { r = idx / BK; kk = idx % BK; }
            As[kk][r] = ra[e];
        }
#pragma unroll
        for (int e = 0; e < (BN * BK) / NT; ++e) {
            const int idx = tid + e * NT;
            int c, kk;
            if (p.tb) { c = idx / BK; kk = idx % BK; } else { kk = idx / BN; c = idx % BN; }
            Bs[kk][c] = rb[e];
        }
        __syncthreads();
        if (k0 + BK < kend) load_tiles(k0 + BK);
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float av[TM], bv[TM];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float4 a = *reinterpret_cast<const float4 *>(&As[kk][ty * 4 + h * (BT / 2)]);
                const float4 b = *reinterpret_cast<const float4 *>(&Bs[kk][tx * 4 + h * (BT / 2)]);
                av[4 * h] = a.x; av[4 * h + 1] = a.y; av[4 * h + 2] = a.z; av[4 * h + 3] = a.w;
                bv[4 * h] = b.x; bv[4 * h + 1] = b.y; bv[4 * h + 2] = b.z; bv[4 * h + 3] = b.w;
            }
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TM; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    pdl_launch_next();
    // epilogue: with beta != 0 every read of C is issued before the first write (one round
    // trip instead of one per element)
    if (p.beta != 0.f) {
#pragma unroll
        for (int i = 0; i < TM; ++i) {
            const int gi = i0 + ty * 4 + (i & 3) + (i >> 2) * (BT / 2);
#pragma unroll
            for (int j = 0; j < TM; ++j) {
                const int gj = j0 + tx * 4 + (j & 3) + (j >> 2) * (BT / 2);
                const bool ok = gi < p.M && gj < p.N && !(p.c_upper && gj < gi);
                acc[i][j] = p.alpha * acc[i][j] +
                            (ok ? p.beta * p.C[(long long)gi * p.ldc + gj] : 0.f);
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TM; ++j) acc[i][j] *= p.alpha;
    }
#pragma unroll
    for (int i = 0; i < TM; ++i) {
        const int gi = i0 + ty * 4 + (i & 3) + (i >> 2) * (BT / 2);
        if (gi >= p.M) continue;
#pragma unroll
        for (int j = 0; j < TM; ++j) {
            const int gj = j0 + tx * 4 + (j & 3) + (j >> 2) * (BT / 2);
            if (gj >= p.N || (p.c_upper && gj < gi)) continue;
            p.C[(long long)gi * p.ldc + gj] = acc[i][j];
        }
    }
}

// Products with M, N, K <= 128 (the blocked factor's 128 x 128 x 128 steps on its serial
// chain): SMALL_T x SMALL_T output tiles (64 CTAs for 128 x 128), the tile's whole K range staged
// at once, one output per thread, summed over k in ascending order as gemm_simt_kernel does (the
// results are the same bit for bit). Small tiles spread the loads over more SMs: the chain's
// products are latency, and 16 x 16 tiles took the factor from 4.0 to 3.65 ms against 32 x 32.
constexpr int SMALL_T = 16, SMALL_K = 128, SMALL_NT = SMALL_T * SMALL_T;
template <typename TA, typename TB>
__global__ __launch_bounds__(SMALL_NT) void gemm_small_kernel(GemmArgs<TA, TB> p) {
    const int i0 = blockIdx.y * SMALL_T, j0 = blockIdx.x * SMALL_T;
    if (p.c_upper && i0 >= j0 + SMALL_T) return;
    pdl_wait_prev();
    if (p.skip && *p.skip) return;
    __shared__ __align__(16) float As[SMALL_K][SMALL_T + 4];  // op(A)[i0 + r, k] at As[k][r]
    __shared__ __align__(16) float Bs[SMALL_K][SMALL_T + 4];  // op(B)[k, j0 + c] at Bs[k][c]
    const int tid = threadIdx.x;
    const int K = p.K;
    // all loads of a thread go out before the first store to shared memory
    constexpr int PER = SMALL_T * SMALL_K / SMALL_NT;
    float va[PER], vb[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int idx = tid + SMALL_NT * e;
        int r, kk;
        if (p.ta) { kk = idx / SMALL_T; r = idx % SMALL_T; } else { r = idx / K; kk = idx % K; }
        const int gi = i0 + r;
        va[e] = 0.f;
        if (idx < SMALL_T * K && gi < p.M && (!p.a_upper || kk >= gi) && (!p.a_lower || kk <= gi))
            va[e] = to_f32(p.ta ? p.A[(long long)kk * p.lda + gi] : p.A[(long long)gi * p.lda + kk]);
        int c, kb;
        if (p.tb) { c = idx / K; kb = idx % K; } else { kb = idx / SMALL_T; c = idx % SMALL_T; }
        const int gj = j0 + c;
        vb[e] = 0.f;
        if (idx < SMALL_T * K && gj < p.N && (!p.b_upper || kb <= gj) && (!p.b_lower || kb >= gj))
            vb[e] = to_f32(p.tb ? p.B[(long long)gj * p.ldb + kb] : p.B[(long long)kb * p.ldb + gj]);
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) {
        const int idx = tid + SMALL_NT * e;
        if (idx >= SMALL_T * K) break;
        int r, kk, c, kb;
        if (p.ta) { kk = idx / SMALL_T; r = idx % SMALL_T; } else { r = idx / K; kk = idx % K; }
        if (p.tb) { c = idx / K; kb = idx % K; } else { kb = idx / SMALL_T; c = idx % SMALL_T; }
        As[kk][r] = va[e];
        Bs[kb][c] = vb[e];
    }
    __syncthreads();
    const int tx = tid % SMALL_T, ty = tid / SMALL_T;
    float acc = 0.f;
#pragma unroll 8
    for (int kk = 0; kk < K; ++kk) acc = fmaf(As[kk][ty], Bs[kk][tx], acc);
    pdl_launch_next();
    const int gi = i0 + ty, gj = j0 + tx;
    if (gi < p.M && gj < p.N && !(p.c_upper && gj < gi)) {
        float *c = p.C + (long long)gi * p.ldc + gj;
        *c = p.beta != 0.f ? p.alpha * acc + p.beta * *c : p.alpha * acc;
    }
}

template <typename TA, typename TB>
inline int gemm_simt(const GemmArgs<TA, TB> &p, cudaStream_t s) {
    if (p.M <= 0 || p.N <= 0) return GPTQ_OK;
    // fewer than ~one 128-tile wave: use 64 x 64 tiles for four times the CTAs
    KtSpan span(s, p.skip != nullptr);
    int st;
    if (p.M <= 128 && p.N <= 128 && p.K <= SMALL_K) {
        dim3 grid(ceil_div(p.N, SMALL_T), ceil_div(p.M, SMALL_T));
        st = launch_kernel(gemm_small_kernel<TA, TB>, grid, dim3(SMALL_NT), 0, s, p.pdl != 0, p);
    } else if ((long long)ceil_div(p.M, 128) * ceil_div(p.N, 128) < 148) {
        dim3 grid(ceil_div(p.N, 64), ceil_div(p.M, 64));
        st = launch_kernel(gemm_simt_kernel<TA, TB, 64>, grid, dim3(simt::NT), 0, s, p.pdl != 0, p);
    } else {
        dim3 grid(ceil_div(p.N, 128), ceil_div(p.M, 128));
        st = launch_kernel(gemm_simt_kernel<TA, TB, 128>, grid, dim3(simt::NT), 0, s, p.pdl != 0, p);
    }
    span.done(KT_SIMT, p);
    return st;
}

template <typename TA, typename TB>
inline GemmArgs<TA, TB> gemm_args(int M, int N, int K, const TA *A, long long lda, int ta,
                                  const TB *B, long long ldb, int tb, float *C, long long ldc,
                                  float alpha, float beta) {
    GemmArgs<TA, TB> p;
    p.M = M; p.N = N; p.K = K;
    p.A = A; p.lda = lda; p.ta = ta;
    p.B = B; p.ldb = ldb; p.tb = tb;
    p.C = C; p.ldc = ldc;
    p.alpha = alpha; p.beta = beta;
    p.c_upper = 0; p.a_upper = 0; p.b_upper = 0; p.a_lower = 0; p.b_lower = 0;
    p.max_ctas = 0;
    p.pdl = 0;
    p.skip = nullptr;
    p.a_lo = nullptr;
    p.b_lo = nullptr;
    p.b_full = nullptr;
    p.ldb_full = 0;
    return p;
}

template <typename T> __device__ __forceinline__ double to_f64(T x) { return (double)x; }
template <> __device__ __forceinline__ double to_f64<__nv_bfloat16>(__nv_bfloat16 x) {
    return (double)__bfloat162float(x);
}

// Optional epilogue of the fp64-accumulating GEMM:
//   C(i,j) = alpha * acc + beta * Cin(i,j) + (i == j ? *diag : 0), written only for j >= i
//   when c_upper is set. Cin may alias C.
struct F64Epilogue {
    const float *Cin = nullptr;
    long long ldcin = 0;
    double beta = 0.0;
    const float *diag = nullptr;
    int c_upper = 0;
    const int *skip = nullptr;   // when set and *skip != 0 the launch does nothing
};

// C = alpha * op(A) op(B) (+ epilogue) accumulated in fp64 (64 x 64 tiles, 4 x 4 per thread).
// For the products whose result is a small difference of large numbers or must keep the weak
// directions of an ill-conditioned block: the orthonormalisation and Rayleigh-Ritz steps and
// the Schur complement of the intrinsic-LoRA factor. The K loop stages 32-deep slabs through
// shared memory with the next slab's global loads in flight. With gridDim.z > 1 the K range
// is split: split z writes its fp64 partial sums to part[z] (M x N, dense) and
// f64acc_reduce_kernel adds the splits in order and applies the epilogue.
constexpr int F64_T = 64, F64_BK = 32;

template <typename TA, typename TB, typename TC>
__global__ __launch_bounds__(256) void gemm_f64acc_kernel(int M, int N, int K, const TA *A,
                                                          long long lda, int ta, const TB *B,
                                                          long long ldb, int tb, TC *C,
                                                          long long ldc, double alpha,
                                                          int b_upper, F64Epilogue ep,
                                                          double *part, int kchunk) {
    constexpr int T = F64_T, BK = F64_BK, PER = T * BK / 256;  // 8 elements per thread
    pdl_wait_prev();
    pdl_launch_next();
    if (ep.skip && *ep.skip) return;
    __shared__ double As[BK][T + 1];
    __shared__ double Bs[BK][T + 1];
    const int i0 = blockIdx.y * T, j0 = blockIdx.x * T;
    if (ep.c_upper && i0 >= j0 + T) return;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    double acc[4][4] = {};
    int kbeg = blockIdx.z * kchunk, kend = min(K, kbeg + kchunk);
    if (b_upper) kend = min(kend, j0 + T);
    double ra[PER], rb[PER];
    auto load = [&](int k0) {
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int idx = tid + 256 * e;
            int r, kk;
            if (ta) { kk = idx / T; r = idx % T; } else { r = idx / BK; kk = idx % BK; }
            const int gi = i0 + r, gk = k0 + kk;
            ra[e] = (gi < M && gk < kend)
                        ? to_f64(ta ? A[(long long)gk * lda + gi] : A[(long long)gi * lda + gk])
                        : 0.0;
            int c;
            if (tb) { c = idx / BK; kk = idx % BK; } else { kk = idx / T; c = idx % T; }
            const int gj = j0 + c, gk2 = k0 + kk;
            rb[e] = (gj < N && gk2 < kend && (!b_upper || gk2 <= gj))
                        ? to_f64(tb ? B[(long long)gj * ldb + gk2] : B[(long long)gk2 * ldb + gj])
                        : 0.0;
        }
    };
    if (kbeg < kend) load(kbeg);
    for (int k0 = kbeg; k0 < kend; k0 += BK) {
#pragma unroll
        for (int e = 0; e < PER; ++e) {
            const int idx = tid + 256 * e;
            if (ta) As[idx / T][idx % T] = ra[e]; else As[idx % BK][idx / BK] = ra[e];
            if (tb) Bs[idx % BK][idx / BK] = rb[e]; else Bs[idx / T][idx % T] = rb[e];
        }
        __syncthreads();
        if (k0 + BK < kend) load(k0 + BK);  // next slab in flight during the FMAs
#pragma unroll 8
        for (int kk = 0; kk < BK; ++kk) {
            double a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { a[u] = As[kk][ty + 16 * u]; b[u] = Bs[kk][tx + 16 * u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
    if (part) {
        double *P = part + (long long)blockIdx.z * M * N;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int gi = i0 + ty + 16 * u;
            if (gi >= M) continue;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const int gj = j0 + tx + 16 * v;
                if (gj < N) P[(long long)gi * N + gj] = acc[u][v];
            }
        }
        return;
    }
    const double dg = ep.diag ? (double)*ep.diag : 0.0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int gi = i0 + ty + 16 * u;
        if (gi >= M) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int gj = j0 + tx + 16 * v;
            if (gj >= N || (ep.c_upper && gj < gi)) continue;
            double val = alpha * acc[u][v];
            if (ep.Cin) val += ep.beta * (double)ep.Cin[(long long)gi * ep.ldcin + gj];
            if (gi == gj) val += dg;
            C[(long long)gi * ldc + gj] = (TC)val;
        }
    }
}

// The same product for A not transposed and M >= 128: 128 x 64 tiles, 256 threads of 8 x 4
// outputs each (a thread's 8 rows are contiguous, so its A values come as 16-byte shared loads
// and every shared load feeds four fp64 FMAs), 16-deep K slabs double-buffered in shared memory
// with the next slab's global loads in flight. B may be transposed; C may be upper (c_upper).
constexpr int F64B_M = 128, F64B_N = 64, F64B_K = 16;

template <typename TA, typename TB, typename TC>
__global__ __launch_bounds__(256, 2) void gemm_f64acc_big_kernel(
    int M, int N, int K, const TA *A, long long lda, const TB *B, long long ldb, int tb, TC *C,
    long long ldc, double alpha, F64Epilogue ep, double *part, int kchunk) {
    pdl_wait_prev();
    pdl_launch_next();
    if (ep.skip && *ep.skip) return;
    __shared__ __align__(16) double As[2][F64B_K][F64B_M];
    __shared__ __align__(16) double Bs[2][F64B_K][F64B_N];
    const int i0 = blockIdx.y * F64B_M, j0 = blockIdx.x * F64B_N;
    if (ep.c_upper && i0 >= j0 + F64B_N) return;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int kbeg = blockIdx.z * kchunk, kend = min(K, kbeg + kchunk);
    // A slab: row ar = tid / 2, k offsets 8 * (tid % 2) .. + 7
    const int ar = tid >> 1, ak = (tid & 1) * 8;
    // B slab (not transposed): k = tid / 16, columns 4 * (tid % 16) .. + 3;
    // (transposed): column = tid / 4, k offsets 4 * (tid % 4) .. + 3
    const int bk_n = tid >> 4, bn_n = (tid & 15) * 4;
    const int bn_t = tid >> 2, bk_t = (tid & 3) * 4;
    double ra[8], rb[4];
    auto load = [&](int k0) {
        const int gi = i0 + ar;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const int gk = k0 + ak + e;
            ra[e] = (gi < M && gk < kend) ? to_f64(A[(long long)gi * lda + gk]) : 0.0;
        }
        if (!tb) {
            const int gk = k0 + bk_n;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int gj = j0 + bn_n + e;
                rb[e] = (gj < N && gk < kend) ? to_f64(B[(long long)gk * ldb + gj]) : 0.0;
            }
        } else {
            const int gj = j0 + bn_t;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int gk = k0 + bk_t + e;
                rb[e] = (gj < N && gk < kend) ? to_f64(B[(long long)gj * ldb + gk]) : 0.0;
            }
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int e = 0; e < 8; ++e) As[buf][ak + e][ar] = ra[e];
        if (!tb) {
#pragma unroll
            for (int e = 0; e < 4; ++e) Bs[buf][bk_n][bn_n + e] = rb[e];
        } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) Bs[buf][bk_t + e][bn_t] = rb[e];
        }
    };
    double acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    int buf = 0;
    if (kbeg < kend) {
        load(kbeg);
        store(0);
    }
    __syncthreads();
    for (int k0 = kbeg; k0 < kend; k0 += F64B_K) {
        const bool more = k0 + F64B_K < kend;
        if (more) load(k0 + F64B_K);   // in flight during the FMAs
#pragma unroll
        for (int kk = 0; kk < F64B_K; ++kk) {
            double av[8], bv[4];
            const double2 *ap = reinterpret_cast<const double2 *>(&As[buf][kk][ty * 8]);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const double2 t = ap[h];
                av[2 * h] = t.x;
                av[2 * h + 1] = t.y;
            }
#pragma unroll
            for (int b = 0; b < 4; ++b) bv[b] = Bs[buf][kk][tx + 16 * b];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fma(av[a], bv[b], acc[a][b]);
        }
        if (more) store(buf ^ 1);
        __syncthreads();
        buf ^= 1;
    }
    if (part) {
        double *P = part + (long long)blockIdx.z * M * N;
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int gi = i0 + ty * 8 + a;
            if (gi >= M) continue;
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const int gj = j0 + tx + 16 * b;
                if (gj < N) P[(long long)gi * N + gj] = acc[a][b];
            }
        }
        return;
    }
    const double dg = ep.diag ? (double)*ep.diag : 0.0;
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int gi = i0 + ty * 8 + a;
        if (gi >= M) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int gj = j0 + tx + 16 * b;
            if (gj >= N || (ep.c_upper && gj < gi)) continue;
            double val = alpha * acc[a][b];
            if (ep.Cin) val += ep.beta * (double)ep.Cin[(long long)gi * ep.ldcin + gj];
            if (gi == gj) val += dg;
            C[(long long)gi * ldc + gj] = (TC)val;
        }
    }
}

// C = alpha * sum_z part[z] (+ epilogue): the splits added in order, so the result does not
// depend on scheduling.
template <typename TC>
__global__ void f64acc_reduce_kernel(int M, int N, int splits, const double *part, TC *C,
                                     long long ldc, double alpha, F64Epilogue ep) {
    pdl_wait_prev();
    pdl_launch_next();
    if (ep.skip && *ep.skip) return;
    const long long total = (long long)M * N;
    const double dg = ep.diag ? (double)*ep.diag : 0.0;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int gi = (int)(idx / N), gj = (int)(idx % N);
        if (ep.c_upper && gj < gi) continue;
        double acc = 0.0;
        for (int z = 0; z < splits; ++z) acc += part[(long long)z * total + idx];
        double val = alpha * acc;
        if (ep.Cin) val += ep.beta * (double)ep.Cin[(long long)gi * ep.ldcin + gj];
        if (gi == gj) val += dg;
        C[(long long)gi * ldc + gj] = (TC)val;
    }
}

// Scratch for split-K: `part` holds part_elems doubles (nullptr: no split).
struct F64Split {
    double *part = nullptr;
    size_t part_elems = 0;
};

template <typename TA, typename TB, typename TC>
inline int gemm_f64acc(int M, int N, int K, const TA *A, long long lda, int ta, const TB *B,
                       long long ldb, int tb, TC *C, long long ldc, double alpha, cudaStream_t s,
                       int b_upper = 0, F64Epilogue ep = F64Epilogue(), F64Split sp = F64Split()) {
    if (M <= 0 || N <= 0) return GPTQ_OK;
    const int sms = device_sm_count();
    if (!ta && !b_upper && M >= F64B_M && N >= 32) {
        // large products: 128 x 64 tiles, split K below two resident CTAs per SM
        dim3 g2(ceil_div(N, F64B_N), ceil_div(M, F64B_M), 1);
        const long long tiles = (long long)g2.x * g2.y;
        int splits = 1;
        if (sp.part && tiles < 2LL * sms && K >= 1024) {
            splits = (int)((2LL * sms + tiles - 1) / tiles);
            if (splits > K / 256) splits = K / 256;
            if (splits > 16) splits = 16;
            while (splits > 1 && (size_t)splits * M * N > sp.part_elems) --splits;
        }
        int kchunk = K;
        if (splits > 1) {
            kchunk = ceil_div(ceil_div(K, splits), F64B_K) * F64B_K;
            splits = ceil_div(K, kchunk);
        }
        g2.z = splits;
        if (int st = launch_kernel(gemm_f64acc_big_kernel<TA, TB, TC>, g2, dim3(256), 0, s, true,
                                   M, N, K, A, lda, B, ldb, tb, C, ldc, alpha, ep,
                                   splits > 1 ? sp.part : nullptr, kchunk))
            return st;
        if (splits > 1) {
            const long long total = (long long)M * N;
            const int blocks = (int)((total + 255) / 256 < 4LL * sms ? (total + 255) / 256 : 4LL * sms);
            return launch_kernel(f64acc_reduce_kernel<TC>, dim3(blocks), dim3(256), 0, s, true, M, N,
                                 splits, (const double *)sp.part, C, ldc, alpha, ep);
        }
        return GPTQ_OK;
    }
    dim3 grid(ceil_div(N, F64_T), ceil_div(M, F64_T), 1);
    // split K when the output tiles fill less than two waves and K is long
    const long long tiles = (long long)grid.x * grid.y;
    int splits = 1;
    if (sp.part && tiles < 2LL * sms && K >= 2048) {
        splits = (int)((2LL * sms + tiles - 1) / tiles);
        if (splits > K / 512) splits = K / 512;
        if (splits > 16) splits = 16;
        while (splits > 1 && (size_t)splits * M * N > sp.part_elems) --splits;
    }
    int kchunk = K;
    if (splits > 1) {
        kchunk = ceil_div(ceil_div(K, splits), F64_BK) * F64_BK;
        splits = ceil_div(K, kchunk);
    }
    grid.z = splits;
    if (int st = launch_kernel(gemm_f64acc_kernel<TA, TB, TC>, grid, dim3(256), 0, s, true, M, N, K,
                               A, lda, ta, B, ldb, tb, C, ldc, alpha, b_upper, ep,
                               splits > 1 ? sp.part : nullptr, kchunk))
        return st;
    if (splits > 1) {
        const long long total = (long long)M * N;
        const int blocks = (int)((total + 255) / 256 < 4LL * sms ? (total + 255) / 256 : 4LL * sms);
        return launch_kernel(f64acc_reduce_kernel<TC>, dim3(blocks), dim3(256), 0, s, true, M, N,
                             splits, (const double *)sp.part, C, ldc, alpha, ep);
    }
    return GPTQ_OK;
}

// Copy the upper triangle of an n x n matrix onto its lower triangle (32x32 smem tiles).
__global__ void mirror_upper_kernel(float *H, long long ld, int n) {
    __shared__ float t[32][33];
    const int bi = blockIdx.y, bj = blockIdx.x;  // destination tile (bi, bj) with bi >= bj
    if (bi < bj) return;
    const int tx = threadIdx.x, ty = threadIdx.y;  // 32 x 8
    for (int y = ty; y < 32; y += 8) {
        const int r = bj * 32 + y, c = bi * 32 + tx;  // source: upper tile (bj, bi)
        if (r < n && c < n) t[y][tx] = H[(long long)r * ld + c];
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
        const int r = bi * 32 + y, c = bj * 32 + tx;
        if (r < n && c < n && r > c) H[(long long)r * ld + c] = t[tx][y];
    }
}

inline int mirror_upper(float *H, long long ld, int n, cudaStream_t s) {
    dim3 grid(ceil_div(n, 32), ceil_div(n, 32));
    mirror_upper_kernel<<<grid, dim3(32, 8), 0, s>>>(H, ld, n);
    return launch_status();
}

}  // namespace gptq
