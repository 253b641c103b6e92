// Top eigenpairs of a small dense symmetric matrix (p <= 128), in fp64, in one CTA.
//
// GPTQ-intrinsic LoRA summary, "Method" part 2: L = V_r, the top-r right singular vectors of
// X. The device finds them by subspace iteration (il.cuh); each Rayleigh-Ritz step needs the
// top-r eigenpairs of the p x p projected matrix T = Y^T H Y. Textbook route, all of it in
// shared memory of one CTA:
//   1. Householder tridiagonalization T = Q Tri Q^T (Golub & Van Loan, "Matrix
//      Computations", section 8.3.1): for k = 0 .. p-3 the reflector H_k = I - tau v v^T maps
//      row k right of the diagonal onto alpha e_1; the trailing block B becomes H_k B H_k by
//      the rank-2 update B - v w^T - w v^T with w = tau B v - (tau^2 / 2)(v^T B v) v.
//   2. Eigenvalues of Tri by multisection on Sturm counts (Wilkinson's bisection, MS_LANES
//      points per round): the number of sign changes of the leading principal minors p_j(x),
//      p_j = (d_j - x) p_{j-1} - e_{j-1}^2 p_{j-2}, is the number of eigenvalues below x.
//   3. Eigenvectors of Tri from the twisted factorization (Dhillon / Parlett's "getvec"):
//      with the forward pivots D+_j = (d_j - lambda) - e_{j-1}^2 / D+_{j-1} and the backward
//      ones D-_j = (d_j - lambda) - e_j^2 / D-_{j+1}, gamma_j = D+_j + D-_j - (d_j - lambda)
//      is smallest where the eigenvector is large; x solves (Tri - lambda) x = gamma_k e_k.
//   4. Back-transformation Q x = H_0 H_1 ... H_{p-3} x.
// Outputs: evals[0 .. r) in decreasing order, Qout (p x r, row-major) the unit eigenvectors.
#pragma once

#include "common.cuh"

namespace gptq {

constexpr int EIG_MAXP = 128;
constexpr int EIG_THREADS = 512;
constexpr int EIG_WARPS = EIG_THREADS / 32;
constexpr int TRI_A = EIG_MAXP / EIG_WARPS;   // rows per thread in the tridiagonalization
constexpr int TRI_B = EIG_MAXP / 32;          // columns per thread
constexpr int TW_BATCH = 2 * EIG_WARPS;       // eigenvectors per twisted-factorization batch

// Shared memory: the Householder vectors packed (v_k, k = 0 .. p-3, has p-k-1 entries), two
// double-buffered vectors (v and p of the current step), d, e, e^2, tau, the pivots of one
// batch of eigenvectors (2p each) and a few scalars.
inline size_t eig_smem(int p) {
    return sizeof(double) * ((size_t)p * (p - 1) / 2 + 4 * (size_t)p + 4 * (size_t)p +
                             (size_t)TW_BATCH * 2 * p + 8);
}

__device__ __forceinline__ double warp_sum_all(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sturm count: the number of eigenvalues of the tridiagonal (d, e2 = e^2) below x, from the
// signs of p_j(x) (p_{-1} = 1; a zero counts as a change of sign and is replaced by a tiny
// value of the opposite sign, so that a split tridiagonal does not carry the zero on). The
// pair (p_j, p_{j-1}) is rescaled every 8 steps so that it stays in range (the recurrence is
// homogeneous in the pair).
__device__ __forceinline__ int sturm_count(const double *d, const double *e2, int p, double x) {
    double pm = 1.0, pc = d[0] - x;
    if (pc == 0.0) pc = -1e-300;
    int cnt = __double2hiint(pc) < 0;
    for (int j0 = 1; j0 < p; j0 += 8) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = j0 + u;
            if (j < p) {
                double pn = fma(d[j] - x, pc, -e2[j - 1] * pm);
                pn = pn == 0.0 ? (__double2hiint(pc) < 0 ? 1e-300 : -1e-300) : pn;
                cnt += (int)((unsigned)(__double2hiint(pn) ^ __double2hiint(pc)) >> 31);
                pm = pc;
                pc = pn;
            }
        }
        const double mx = fmax(fabs(pc), fabs(pm));
        if (mx > 1e120) { pc *= 1e-120; pm *= 1e-120; }
        else if (mx < 1e-120) { pc *= 1e120; pm *= 1e120; }
    }
    return cnt;
}

// Lanes per eigenvalue in the multisection: each round the group evaluates the Sturm count at
// MS_LANES interior points of its interval and keeps the one subinterval that holds the
// eigenvalue (a factor MS_LANES + 1 per round).
constexpr int MS_LANES = 8;
constexpr int MS_ROUNDS = 17;   // 9^17 > 1e16: from the Gershgorin width to ~1e-16 of it

__device__ __forceinline__ double safe_pivot(double D, double pivmin) {
    return fabs(D) < pivmin ? (D < 0.0 ? -pivmin : pivmin) : D;
}

// skip: when not null and *skip != 0 the kernel returns at once (an iteration that is no
// longer needed).
__global__ __launch_bounds__(EIG_THREADS) void sym_eig_top_kernel(const double *Tin, int p, int r,
                                                                  double *evals, double *Qout,
                                                                  const int *skip) {
    pdl_wait_prev();
    pdl_launch_next();
    if (skip && *skip) return;
    extern __shared__ __align__(16) double esm[];
    double *Vh = esm;                              // packed Householder vectors
    double *xbuf = Vh + p * (p - 1) / 2;           // 2 x p
    double *pbuf = xbuf + 2 * p;                   // 2 x p
    double *d = pbuf + 2 * p;
    double *e = d + p;
    double *e2 = e + p;
    double *tau = e2 + p;
    double *Dpm = tau + p;                         // TW_BATCH x 2p
    double *scal = Dpm + TW_BATCH * 2 * p;         // [0] lo, [1] hi, [2] |T| bound
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // ---- 1. tridiagonalization with the matrix in registers: thread (warp, lane) holds rows
    // warp + 16 a and columns lane + 32 b. v_k goes to Vh at offset k (p - 1) - k (k - 1) / 2.
    double M[TRI_A][TRI_B];
#pragma unroll
    for (int a = 0; a < TRI_A; ++a)
#pragma unroll
        for (int b = 0; b < TRI_B; ++b) {
            const int i = warp + EIG_WARPS * a, j = lane + 32 * b;
            M[a][b] = (i < p && j < p)
                          ? 0.5 * (Tin[(long long)i * p + j] + Tin[(long long)j * p + i]) : 0.0;
        }
    for (int k = 0; k + 2 < p; ++k) {
        const int buf = k & 1;
        double *xv = xbuf + buf * p, *pv = pbuf + buf * p;
        if (warp == k % EIG_WARPS) {
            // the owner of row k forms the reflector that maps row k right of the diagonal
            // onto alpha e_1 and publishes v (absolute column indices), tau, alpha and d_k
            const int oa = k / EIG_WARPS;
            double xr[TRI_B];
#pragma unroll
            for (int b = 0; b < TRI_B; ++b) {
                double v = 0.0;
#pragma unroll
                for (int a = 0; a < TRI_A; ++a) if (a == oa) v = M[a][b];
                xr[b] = v;
            }
            double ss = 0.0, x0 = 0.0, dk = 0.0;
#pragma unroll
            for (int b = 0; b < TRI_B; ++b) {
                const int j = lane + 32 * b;
                if (j > k && j < p) ss = fma(xr[b], xr[b], ss);
                if (j == k + 1) x0 = xr[b];
                if (j == k) dk = xr[b];
            }
            ss = warp_sum_all(ss);
            x0 = __shfl_sync(0xffffffffu, x0, (k + 1) & 31);
            const double nrm = sqrt(ss);
            const double alpha = nrm == 0.0 ? 0.0 : (x0 >= 0.0 ? -nrm : nrm);
            const double tk = nrm == 0.0 ? 0.0 : 1.0 / (ss - alpha * x0);
            const double v0 = x0 - alpha;
            double *vk = Vh + (long long)k * (p - 1) - (long long)k * (k - 1) / 2;
#pragma unroll
            for (int b = 0; b < TRI_B; ++b) {
                const int j = lane + 32 * b;
                if (j > k && j < p) {
                    const double v = j == k + 1 ? v0 : xr[b];
                    xv[j] = v;
                    vk[j - k - 1] = v;
                }
            }
            if (lane == (k & 31)) d[k] = dk;
            if (lane == 0) { e[k] = alpha; tau[k] = tk; }
        }
        __syncthreads();
        const double tk = tau[k];
        // row block a holds rows > k only if 16 a + 15 > k; column block b only if 32 b + 31 > k
        const int a0 = k >= EIG_WARPS - 1 ? (k - (EIG_WARPS - 1)) / EIG_WARPS : 0;
        const int b0 = k >= 31 ? (k - 31) / 32 : 0;
        double vc[TRI_B], vr[TRI_A], pr[TRI_A];
#pragma unroll
        for (int b = 0; b < TRI_B; ++b) {
            const int j = lane + 32 * b;
            vc[b] = (j > k && j < p) ? xv[j] : 0.0;
        }
        // p = tau B v over the trailing rows (a row block at or above k has nothing to add)
#pragma unroll
        for (int a = 0; a < TRI_A; ++a) {
            const int i = warp + EIG_WARPS * a;
            const bool live = i > k && i < p;
            vr[a] = live ? xv[i] : 0.0;
            double acc = 0.0;
            if (a >= a0) {
#pragma unroll
                for (int b = 0; b < TRI_B; ++b)
                    if (b >= b0) acc = fma(M[a][b], vc[b], acc);
            }
            pr[a] = live ? acc : 0.0;
        }
        // sum over the 32 lanes: a reduce-scatter (row a's sum ends in lane 4a .. 4a + 3)
        // followed by a broadcast, 8 + 4 + 2 + 1 + 1 exchanges instead of 8 x 5
        {
            double t4[4], t2[2], t1;
            const bool hi16 = lane & 16, hi8 = lane & 8, hi4 = lane & 4;
#pragma unroll
            for (int q = 0; q < 4; ++q) {   // halves exchanged with lane ^ 16
                const double mine = hi16 ? pr[q + 4] : pr[q];
                const double send = hi16 ? pr[q] : pr[q + 4];
                t4[q] = mine + __shfl_xor_sync(0xffffffffu, send, 16);
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const double mine = hi8 ? t4[q + 2] : t4[q];
                const double send = hi8 ? t4[q] : t4[q + 2];
                t2[q] = mine + __shfl_xor_sync(0xffffffffu, send, 8);
            }
            {
                const double mine = hi4 ? t2[1] : t2[0];
                const double send = hi4 ? t2[0] : t2[1];
                t1 = mine + __shfl_xor_sync(0xffffffffu, send, 4);
            }
            t1 += __shfl_xor_sync(0xffffffffu, t1, 2);
            t1 += __shfl_xor_sync(0xffffffffu, t1, 1);
            // lane l now holds the full sum of row block a = 4 (l >> 4 & 1) + 2 (l >> 3 & 1) +
            // (l >> 2 & 1); gather each back to every lane
#pragma unroll
            for (int a = 0; a < TRI_A; ++a) {
                const int src = ((a >> 2) & 1) * 16 + ((a >> 1) & 1) * 8 + (a & 1) * 4;
                pr[a] = __shfl_sync(0xffffffffu, t1, src);
            }
        }
#pragma unroll
        for (int a = 0; a < TRI_A; ++a) {
            pr[a] *= tk;
            const int i = warp + EIG_WARPS * a;
            if (lane == 0 && i > k && i < p) pv[i] = pr[a];
        }
        __syncthreads();
        // K = tau/2 v^T p, w = p - K v; B -= v w^T + w v^T
        double kd = 0.0;
#pragma unroll
        for (int b = 0; b < TRI_B; ++b) {
            const int j = lane + 32 * b;
            if (j > k && j < p) kd = fma(vc[b], pv[j], kd);
        }
        kd = 0.5 * tk * warp_sum_all(kd);
        double wc[TRI_B];
#pragma unroll
        for (int b = 0; b < TRI_B; ++b) {
            const int j = lane + 32 * b;
            wc[b] = (j > k && j < p) ? fma(-kd, vc[b], pv[j]) : 0.0;
        }
#pragma unroll
        for (int a = 0; a < TRI_A; ++a) {
            if (a < a0) continue;
            const double wr = fma(-kd, vr[a], pr[a]);
#pragma unroll
            for (int b = 0; b < TRI_B; ++b)
                if (b >= b0) M[a][b] -= fma(vr[a], wc[b], wr * vc[b]);
        }
    }
    // the last 2 x 2 block
#pragma unroll
    for (int a = 0; a < TRI_A; ++a)
#pragma unroll
        for (int b = 0; b < TRI_B; ++b) {
            const int i = warp + EIG_WARPS * a, j = lane + 32 * b;
            if (p >= 2 && i == p - 2 && j == p - 2) d[p - 2] = M[a][b];
            if (p >= 2 && i == p - 2 && j == p - 1) e[p - 2] = M[a][b];
            if (i == p - 1 && j == p - 1) d[p - 1] = M[a][b];
        }
    __syncthreads();
    if (tid == 0) {
        e[p - 1] = 0.0;
        // Gershgorin interval and a norm bound
        double lo = 1e300, hi = -1e300, tn = 0.0;
        for (int j = 0; j < p; ++j) {
            const double rad = fabs(e[j]) + (j > 0 ? fabs(e[j - 1]) : 0.0);
            lo = fmin(lo, d[j] - rad);
            hi = fmax(hi, d[j] + rad);
            tn = fmax(tn, fabs(d[j]) + rad);
        }
        const double pad = 1e-14 * tn + 1e-300;
        scal[0] = lo - pad;
        scal[1] = hi + pad;
        scal[2] = tn;
    }
    __syncthreads();
    for (int j = tid; j < p; j += EIG_THREADS) e2[j] = e[j] * e[j];
    __syncthreads();

    // ---- 2. eigenvalues c = 0 .. r-1 (decreasing): multisection, MS_LANES lanes per eigenvalue
    const double tnorm = scal[2];
    {
        constexpr int GROUPS = 32 / MS_LANES;
        const int grp = lane / MS_LANES, gl = lane % MS_LANES;
        const unsigned gmask = ((1u << MS_LANES) - 1u) << (grp * MS_LANES);
        for (int c0 = warp * GROUPS; c0 < r; c0 += EIG_WARPS * GROUPS) {
            const int c = c0 + grp;
            const int t = p - 1 - min(c, r - 1);   // ascending index (idle groups repeat r-1)
            double a = scal[0], b = scal[1];
            for (int round = 0; round < MS_ROUNDS; ++round) {
                const double x = a + (b - a) * (double)(gl + 1) / (double)(MS_LANES + 1);
                const bool above = sturm_count(d, e2, p, x) > t;
                const unsigned bits = (__ballot_sync(0xffffffffu, above) & gmask) >> (grp * MS_LANES);
                const int l = bits ? __ffs(bits) - 1 : MS_LANES;
                const double xl = __shfl_sync(0xffffffffu, x, grp * MS_LANES + (l < MS_LANES ? l : 0));
                const double xlm = __shfl_sync(0xffffffffu, x, grp * MS_LANES + (l > 0 ? l - 1 : 0));
                const double na = l == 0 ? a : xlm;
                const double nb = l == MS_LANES ? b : xl;
                a = na;
                b = nb;
            }
            if (gl == 0 && c < r) evals[c] = 0.5 * (a + b);
        }
    }
    __threadfence_block();
    __syncthreads();

    // ---- 3. eigenvectors of the tridiagonal in batches of TW_BATCH, two per warp (lanes 0-1
    // and 2-3 run the forward and backward pivot recurrences, with reciprocals); written to
    // Qout's columns
    const double pivmin = 1e-290 * fmax(1.0, tnorm * tnorm);
    for (int c0 = 0; c0 < r; c0 += TW_BATCH) {
        const int slot = lane >> 1;                  // 0 or 1 for lanes 0-3
        const int bidx = warp * 2 + (slot & 1);
        const int c = c0 + bidx;
        double *Dp = Dpm + bidx * 2 * p, *Dm = Dp + p;
        const bool act = lane < 4 && c < r;
        const double lam = act ? evals[c] : 0.0;
        if (act && (lane & 1) == 0) {
            double D = safe_pivot(d[0] - lam, pivmin);
            Dp[0] = D;
            for (int j = 1; j < p; ++j) {
                D = safe_pivot((d[j] - lam) - e2[j - 1] * __drcp_rn(D), pivmin);
                Dp[j] = D;
            }
        } else if (act) {
            double D = safe_pivot(d[p - 1] - lam, pivmin);
            Dm[p - 1] = D;
            for (int j = p - 2; j >= 0; --j) {
                D = safe_pivot((d[j] - lam) - e2[j] * __drcp_rn(D), pivmin);
                Dm[j] = D;
            }
        }
        __syncwarp();
        // twist index of each of the warp's two eigenvectors: smallest |gamma_j| (first on ties)
        int bi2[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int ch = c0 + warp * 2 + h;
            const double *Dph = Dpm + (warp * 2 + h) * 2 * p, *Dmh = Dph + p;
            const double lh = ch < r ? evals[ch] : 0.0;
            double best = 1e308;
            int bi = 0;
            if (ch < r)
                for (int j = lane; j < p; j += 32) {
                    const double g = fabs(Dph[j] + Dmh[j] - (d[j] - lh));
                    if (g < best) { best = g; bi = j; }
                }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ob = __shfl_xor_sync(0xffffffffu, best, o);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
                if (ob < best || (ob == best && oi < bi)) { best = ob; bi = oi; }
            }
            bi2[h] = bi;
        }
        __syncwarp();
        // x_k = 1; downwards from the twist with D+, upwards with D-; x overwrites the pivots
        const int bi = bi2[slot & 1];
        if (act && (lane & 1) == 0) {
            double x = 1.0;
            for (int j = bi - 1; j >= 0; --j) {
                x = -(e[j] * __drcp_rn(Dp[j])) * x;
                Dp[j] = x;
            }
            Dp[bi] = 1.0;
        } else if (act) {
            double x = 1.0;
            for (int j = bi + 1; j < p; ++j) {
                x = -(e[j - 1] * __drcp_rn(Dm[j])) * x;
                Dm[j] = x;
            }
        }
        __syncwarp();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int ch = c0 + warp * 2 + h;
            if (ch >= r) continue;
            const double *Dph = Dpm + (warp * 2 + h) * 2 * p, *Dmh = Dph + p;
            const int bh = bi2[h];
            double ss = 0.0;
            for (int j = lane; j < p; j += 32) {
                const double x = j <= bh ? Dph[j] : Dmh[j];
                ss += x * x;
            }
            ss = warp_sum_all(ss);
            const double inv = 1.0 / sqrt(ss);
            for (int j = lane; j < p; j += 32)
                Qout[(long long)j * r + ch] = (j <= bh ? Dph[j] : Dmh[j]) * inv;
        }
        __syncwarp();
    }
    __threadfence_block();
    __syncthreads();

    // Eigenvalues closer than 1e-9 |T| (not met with distinct eigenvalues) give nearly the same
    // twisted-factorization vector: warp 0 re-orthogonalizes each against the earlier members
    // of its cluster (Gram-Schmidt in the tridiagonal basis).
    if (warp == 0) {
        const double ctol = 1e-9 * tnorm;
        for (int c = 1; c < r; ++c) {
            int cs = c;
            while (cs > 0 && fabs(evals[cs - 1] - evals[c]) <= ctol) --cs;
            if (cs == c) continue;
            for (int pass = 0; pass < 2; ++pass) {
                for (int c2 = cs; c2 < c; ++c2) {
                    double dt = 0.0;
                    for (int j = lane; j < p; j += 32) dt += Qout[(long long)j * r + c] * Qout[(long long)j * r + c2];
                    dt = warp_sum_all(dt);
                    for (int j = lane; j < p; j += 32) Qout[(long long)j * r + c] -= dt * Qout[(long long)j * r + c2];
                    __syncwarp();
                }
                double ss = 0.0;
                for (int j = lane; j < p; j += 32) ss += Qout[(long long)j * r + c] * Qout[(long long)j * r + c];
                ss = warp_sum_all(ss);
                const double inv = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;
                for (int j = lane; j < p; j += 32) Qout[(long long)j * r + c] *= inv;
                __syncwarp();
            }
        }
    }
    __threadfence_block();
    __syncthreads();

    // ---- 4. back-transformation Q x = H_0 ... H_{p-3} x: groups of 4 lanes hold one
    // eigenvector each (lane g of a group holds entries 4 i + g, i < 32), 8 per warp
    {
        constexpr int GL = 4, PER = EIG_MAXP / GL;   // 32 entries per lane
        const int grp = lane / GL, gl = lane % GL;
        for (int c0 = warp * (32 / GL); c0 < r; c0 += EIG_WARPS * (32 / GL)) {
            const int c = c0 + grp;
            const bool own = c < r;
            double x[PER];
#pragma unroll
            for (int q = 0; q < PER; ++q) {
                const int i = GL * q + gl;
                x[q] = (own && i < p) ? Qout[(long long)i * r + c] : 0.0;
            }
            for (int k = p - 3; k >= 0; --k) {
                const double *vk = Vh + (long long)k * (p - 1) - (long long)k * (k - 1) / 2 - (k + 1);
                const int q0 = (k + 1) / GL;   // entries below q0 * GL are not touched by H_k
                double dot = 0.0;
#pragma unroll
                for (int q = 0; q < PER; ++q) {
                    const int i = GL * q + gl;
                    if (q >= q0 && i > k && i < p) dot = fma(vk[i], x[q], dot);
                }
                dot += __shfl_xor_sync(0xffffffffu, dot, 1);
                dot += __shfl_xor_sync(0xffffffffu, dot, 2);
                const double f = tau[k] * dot;
#pragma unroll
                for (int q = 0; q < PER; ++q) {
                    const int i = GL * q + gl;
                    if (q >= q0 && i > k && i < p) x[q] = fma(-f, vk[i], x[q]);
                }
            }
            if (own)
#pragma unroll
                for (int q = 0; q < PER; ++q) {
                    const int i = GL * q + gl;
                    if (i < p) Qout[(long long)i * r + c] = x[q];
                }
        }
    }
}

// Top r eigenpairs of the symmetric p x p fp64 matrix T (p <= EIG_MAXP, r <= p).
inline int sym_eig_top(const double *T, int p, int r, double *evals, double *Q, const int *skip,
                       cudaStream_t s) {
    if (p < 1 || p > EIG_MAXP || r < 1 || r > p) return GPTQ_ERR_ARG;
    const size_t smem = eig_smem(p);
    GPTQ_SMEM_LIMIT(sym_eig_top_kernel, eig_smem(EIG_MAXP));
    return launch_kernel(sym_eig_top_kernel, dim3(1), dim3(EIG_THREADS), smem, s, true, T, p, r,
                         evals, Q, skip);
}

}  // namespace gptq
