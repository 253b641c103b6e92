// Two-sided adaptive rounding (GPTQ-2D: Cubic-Time Two-Sided Adaptive Rounding).
//
// Round X (m x n) to integers Z under the Gram matrix H (x) G of the vectorised problem.
// With U_G, U_H the upper factors of G^-1 and H^-1 (G^-1 = U_G^T U_G), rounding entry (i, j)
// with error e_ij feeds U_G[i, p] U_H[j, q] e_ij into every later entry (p >= i, q >= j)
// (section 2, Kronecker feedback), so the entries of one anti-diagonal are independent and
// the sweep runs in m + n - 1 stages. Two buffers carry the feedback (section 2, the buffer
// C = L E): errors are pushed down their column into C, and a column buffer value, once final,
// is pushed along its row.
//
// Device organisation (section 2, blocked variant): the matrix is cut into 32 x 32 tiles; the
// tiles of one tile anti-diagonal are independent and are swept by one CTA each. Stages are
// grouped in bands of W tile anti-diagonals: a tile pulls the contributions of the tiles of
// its own band that precede it (small 32 x 32 x 32 products), and at the end of each band the
// band's errors are flushed at once into all later tiles (the banded product of the blocked
// algorithm):
//   Cacc[p, J] += U_G[band rows of J, p]^T E[band rows, J]   (column flush)
//   Xw[I, q]  -= F[I, band cols of I] U_H[band cols, q]       (row flush)
// where F is the final column buffer (C after the entry's own error) and Xw = X minus all
// flushed row pushes. Padded rows / columns (m, n not multiples of 32) carry zero input and
// identity factors; feedback only flows down and right, so they never reach a real entry.
#pragma once

#include <algorithm>
#include <mutex>

#include "common.cuh"

namespace gptq {

constexpr int T2D = 32;             // tile edge
constexpr int T2D_THREADS = 128;    // CTA of the tile sweep and of the flushes
constexpr int T2D_BAND_DEFAULT = 4; // tile anti-diagonals per band
constexpr int T2D_BAND_MAX = 8;

struct Gptq2dArgs {
    float *Xw;          // Mp x Np, ld Np: X minus the flushed row pushes (padding zero)
    float *Cacc;        // Mp x Np, ld Np: flushed column pushes
    float *E;           // Mp x Np, ld Np: errors e_ij
    float *F;           // Mp x Np, ld Np: final column buffer values
    const float *UG;    // Mp x Mp, ld Mp: upper factor of G^-1 (identity on the padding)
    const float *UH;    // Np x Np, ld Np: upper factor of H^-1
    int32_t *Z;         // m x n, ld n: the rounded integers
    float *err;         // optional m x n, ld n: e_ij
    long long Mp, Np;
    int m, n, MT, NT;
};

// Programmatic dependent launch (common.cuh): every kernel of the wavefront lets the next one
// start at once (its independent prologue overlaps this kernel) and waits for the previous
// kernel's completion before it touches anything that kernel wrote.

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// One 32 x 32 fp32 tile (global row pitch ld floats) into shared memory (pitch 32), as 256
// 16-byte copies spread over the CTA's 128 threads.
__device__ __forceinline__ void tile_async(float *dst, const float *src, long long ld) {
    for (int c = threadIdx.x; c < T2D * T2D / 4; c += T2D_THREADS) {
        const int r = c >> 3, q = (c & 7) * 4;
        cp_async16(dst + r * T2D + q, src + r * ld + q);
    }
}

constexpr int T2D_TILE = T2D * T2D;   // floats in one tile
constexpr int UHS_PITCH = T2D + 4;
// dynamic shared memory of the sweep: 10 fixed tiles (Cs, Xs, UGd, the two shifted copies of
// U_H[J, J] with its reciprocals (three tiles), Es, Fs, Zs) and two operand tiles per pulled
// tile (up to W - 1 per direction)
inline size_t gptq2d_sweep_smem(int band) { return sizeof(float) * T2D_TILE * (10 + 4 * (band - 1)); }

// Physical register p of a rotated row holds slot (base + p) % 32; the rows are kept as pairs
// of slots, and rotating the pair array down by R pairs after 2R steps keeps the slot of the
// current step at index 0 .. 2R-1.
template <int R>
__device__ __forceinline__ void rotate_down2(float2 (&x)[T2D / 2]) {
    float2 t[R];
#pragma unroll
    for (int i = 0; i < R; ++i) t[i] = x[i];
#pragma unroll
    for (int i = 0; i < T2D / 2 - R; ++i) x[i] = x[i + R];
#pragma unroll
    for (int i = 0; i < R; ++i) x[T2D / 2 - R + i] = t[i];
}

// ---------------------------------------------------------------------------------------
// Tile sweep of stage S (tiles with I + J = S). One CTA per tile. Tiles of stages [W0, S) are
// pulled; everything before stage W0 has been flushed into Cacc / Xw.
// All operands are copied to shared memory at once; the four warps add the band's earlier
// tiles (pulls), then warp 0 sweeps the tile's 63 anti-diagonals. The error is formed with
// the reciprocals of the two diagonal entries (within a few ulp of the quotient).
// ---------------------------------------------------------------------------------------
constexpr int T2D_UNROLL = 8;

__global__ __launch_bounds__(T2D_THREADS) void gptq2d_sweep_kernel(Gptq2dArgs a, int S, int W0) {
    extern __shared__ __align__(16) float sm[];
    float *Cs = sm, *Xs = sm + T2D_TILE, *UGd = sm + 2 * T2D_TILE;
    // U_H[J, J] with row b shifted left by b: UHs[b][k] = U_H[b, b + k] (zero past the tile),
    // UHs1[b][k] = U_H[b, b + k - 1] (one further right); pitch 36 so that the lanes' 16-byte
    // row reads fall in distinct banks
    float *UHs = sm + 3 * T2D_TILE;
    float *UHs1 = UHs + T2D * UHS_PITCH;
    float *ruh = UHs1 + T2D * UHS_PITCH;                // 1 / U_H[b, b]
    float *Es = sm + 6 * T2D_TILE, *Fs = sm + 7 * T2D_TILE;
    int *Zs = reinterpret_cast<int *>(sm + 8 * T2D_TILE);
    float *P = sm + 10 * T2D_TILE;                      // pulled operand pairs

    const int tid = threadIdx.x;
    const int I = max(0, S - a.NT + 1) + blockIdx.x;
    const int J = S - I;
    const long long r0g = (long long)I * T2D, c0g = (long long)J * T2D;
    const int i_lo = max(0, W0 - J), j_lo = max(0, W0 - I);
    const int nc = I - i_lo, nr = J - j_lo;

    pdl_launch_next();
    // the factors were final before the wavefront began: fetch them first
    tile_async(UGd, a.UG + r0g * a.Mp + r0g, a.Mp);
    float *Pr = P + 2 * nc * T2D_TILE;
    for (int i = 0; i < nc; ++i) {
        const long long k0 = (long long)(i_lo + i) * T2D;
        tile_async(P + (2 * i) * T2D_TILE, a.UG + k0 * a.Mp + r0g, a.Mp);      // U_G[k, p]
    }
    for (int j = 0; j < nr; ++j) {
        const long long k0 = (long long)(j_lo + j) * T2D;
        tile_async(Pr + (2 * j + 1) * T2D_TILE, a.UH + k0 * a.Np + c0g, a.Np); // U_H[k, q]
    }
    for (int t = tid; t < T2D_TILE; t += T2D_THREADS) {
        const int r = t >> 5, k = t & 31;
        const float h = r + k < T2D ? a.UH[(c0g + r) * a.Np + c0g + r + k] : 0.f;
        UHs[r * UHS_PITCH + k] = h;
        UHs1[r * UHS_PITCH + k + 1] = h;
        if (k == 0) {
            ruh[r] = 1.f / h;
            UHs1[r * UHS_PITCH] = 0.f;
            UHs1[r * UHS_PITCH + T2D + 1] = 0.f;
            UHs1[r * UHS_PITCH + T2D + 2] = 0.f;
            UHs1[r * UHS_PITCH + T2D + 3] = 0.f;
        }
    }
    // then what the earlier stages and flushes wrote
    pdl_wait_prev();
    tile_async(Cs, a.Cacc + r0g * a.Np + c0g, a.Np);
    tile_async(Xs, a.Xw + r0g * a.Np + c0g, a.Np);
    for (int i = 0; i < nc; ++i) {
        const long long k0 = (long long)(i_lo + i) * T2D;
        tile_async(P + (2 * i + 1) * T2D_TILE, a.E + k0 * a.Np + c0g, a.Np);   // e[k, q]
    }
    for (int j = 0; j < nr; ++j) {
        const long long k0 = (long long)(j_lo + j) * T2D;
        tile_async(Pr + (2 * j) * T2D_TILE, a.F + r0g * a.Np + k0, a.Np);      // f[p, k]
    }
    cp_async_wait_all();
    __syncthreads();

    const int tx = tid & 31, ty = tid >> 5;   // outputs: rows ty*8 .. +8 of column tx
    if (nc + nr > 0) {
        float cacc[8], vacc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) cacc[i] = vacc[i] = 0.f;
        for (int i = 0; i < nc; ++i) {
            const float *A = P + (2 * i) * T2D_TILE, *B = P + (2 * i + 1) * T2D_TILE;
#pragma unroll 4
            for (int k = 0; k < T2D; ++k) {
                const float b = B[k * T2D + tx];
                const float4 a0 = *reinterpret_cast<const float4 *>(A + k * T2D + ty * 8);
                const float4 a1 = *reinterpret_cast<const float4 *>(A + k * T2D + ty * 8 + 4);
                cacc[0] += a0.x * b; cacc[1] += a0.y * b; cacc[2] += a0.z * b; cacc[3] += a0.w * b;
                cacc[4] += a1.x * b; cacc[5] += a1.y * b; cacc[6] += a1.z * b; cacc[7] += a1.w * b;
            }
        }
        for (int j = 0; j < nr; ++j) {
            const float *A = Pr + (2 * j) * T2D_TILE, *B = Pr + (2 * j + 1) * T2D_TILE;
#pragma unroll 2
            for (int k = 0; k < T2D; k += 4) {
                const float b0 = B[k * T2D + tx], b1 = B[(k + 1) * T2D + tx];
                const float b2 = B[(k + 2) * T2D + tx], b3 = B[(k + 3) * T2D + tx];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 f = *reinterpret_cast<const float4 *>(A + (ty * 8 + i) * T2D + k);
                    vacc[i] += f.x * b0 + f.y * b1 + f.z * b2 + f.w * b3;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            Cs[(ty * 8 + i) * T2D + tx] += cacc[i];
            Xs[(ty * 8 + i) * T2D + tx] -= vacc[i];
        }
        __syncthreads();
    }

    if (ty == 0) {
        // Lane l owns tile row l; slot s % 32 of its rotated arrays holds column (s - l) % 32.
        // Slots are kept in pairs (2P, 2P+1) so that the pushes run as paired FMAs; at odd
        // steps the operand pairs come from copies shifted by one (UHs1, ug1).
        const int l = tx;
        float2 xw2[T2D / 2], cc2[T2D / 2], ug0[T2D / 2], ug1[T2D / 2 + 1];
#pragma unroll
        for (int p = 0; p < T2D; p += 2) {
            const int c0 = (p - l) & 31, c1 = (p + 1 - l) & 31;
            xw2[p >> 1] = make_float2(Xs[l * T2D + c0], Xs[l * T2D + c1]);
            cc2[p >> 1] = make_float2(Cs[l * T2D + c0], Cs[l * T2D + c1]);
        }
        // ugc[d] = U_G[l-d, l] (0 for d = 0 or d > l); ug0 pairs (ugc[2i], ugc[2i+1]),
        // ug1 pairs (ugc[2i-1], ugc[2i]) with ugc[-1] = ugc[32] = 0
        auto ugc = [&](int d) { return (d >= 1 && d < T2D && l >= d) ? UGd[(l - d) * T2D + l] : 0.f; };
#pragma unroll
        for (int i = 0; i < T2D / 2; ++i) ug0[i] = make_float2(ugc(2 * i), ugc(2 * i + 1));
#pragma unroll
        for (int i = 0; i <= T2D / 2; ++i) ug1[i] = make_float2(ugc(2 * i - 1), ugc(2 * i));
        const float ugd = UGd[l * T2D + l];
        const float rug = 1.f / ugd;
        int bad = 0;
#pragma unroll 1
        for (int base = 0; base < 2 * T2D; base += T2D_UNROLL) {
#pragma unroll
            for (int u = 0; u < T2D_UNROLL; ++u) {
                const int b = base + u - l;                // this lane's column at this step
                const bool act = (unsigned)b < (unsigned)T2D;
                const int bc = act ? b : 0;
                const bool odd = u & 1;
                // uh pairs: even steps (U_H[b, b+2i], U_H[b, b+2i+1]); odd steps shifted by one
                float2 uh[T2D / 2 + 2];
                const float *uhrow = (odd ? UHs1 : UHs) + bc * UHS_PITCH;
#pragma unroll
                for (int i4 = 0; i4 < (odd ? 9 : 8); ++i4) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(uhrow + 4 * i4);
                    uh[2 * i4] = make_float2(t4.x, t4.y);
                    uh[2 * i4 + 1] = make_float2(t4.z, t4.w);
                }
                const float uhd = odd ? uh[0].y : uh[0].x;
                const float xu = (u & 1) ? xw2[u >> 1].y : xw2[u >> 1].x;
                const float cu = (u & 1) ? cc2[u >> 1].y : cc2[u >> 1].x;
                const float rinv = rug * ruh[bc];
                const float v = xu - cu * uhd;
                const float z = rintf(v);
                const float e = act ? (v - z) * rinv : 0.f;
                const float cf = act ? cu + ugd * e : 0.f;
                if (act) {
                    bad |= !isfinite(v);
                    Zs[l * T2D + b] = __float2int_rn(z);
                    Es[l * T2D + b] = e;
                    Fs[l * T2D + b] = cf;
                }
                const float2 ncf = make_float2(-cf, -cf);
#pragma unroll
                for (int i = 0; i < T2D / 2; ++i) {
                    // the pair holding the next step's slot first (the next decision waits on
                    // it), then the rest. Slots 2P, 2P+1 are d0 = (2P - u) % 32 and d1 =
                    // (d0 + 1) % 32 steps ahead; d = 0 is the slot just consumed (its weights
                    // are zero or unused)
                    const int P = (((u + 1) >> 1) + i) & (T2D / 2 - 1);
                    const int d0 = (2 * P - u) & 31, d1 = (d0 + 1) & 31;
                    const float e0 = d0 ? __shfl_up_sync(0xffffffffu, e, d0) : e;
                    const float e1 = d1 ? __shfl_up_sync(0xffffffffu, e, d1) : e;
                    // error down the column (lane l - d decided column b + d)
                    cc2[P] = __ffma2_rn(odd ? ug1[(d0 + 1) >> 1] : ug0[d0 >> 1], make_float2(e0, e1), cc2[P]);
                    // final column buffer value along the own row
                    xw2[P] = __ffma2_rn(ncf, odd ? uh[(d0 + 1) >> 1] : uh[d0 >> 1], xw2[P]);
                }
            }
            rotate_down2<T2D_UNROLL / 2>(xw2);
            rotate_down2<T2D_UNROLL / 2>(cc2);
        }
        if (bad) report(GPTQ_ERR_NONFINITE, r0g + l);
    }
    __syncthreads();
    for (int t = tid; t < T2D_TILE; t += T2D_THREADS) {
        const int r = t >> 5, c = t & 31;
        const long long idx = (r0g + r) * a.Np + c0g + c;
        a.E[idx] = Es[t];
        a.F[idx] = Fs[t];
        const long long p = r0g + r, q = c0g + c;
        if (p < a.m && q < a.n) {
            a.Z[p * a.n + q] = Zs[t];
            if (a.err) a.err[p * a.n + q] = Es[t];
        }
    }
}

// 16-byte copy that writes zeros instead when `valid` is false (src must still be mapped).
__device__ __forceinline__ void cp_async16_or_zero(void *smem_dst, const void *gmem_src, bool valid) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(gmem_src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

constexpr int FLUSH_THREADS = 256;
constexpr int CF_ROWS = 128;   // column flush: target rows per CTA (x 32 columns of the strip)
constexpr int RF_COLS = 256;   // row flush: target columns per CTA (x 32 rows of the strip)
inline size_t gptq2d_col_flush_smem(int band) {
    return sizeof(float) * ((size_t)band * T2D * T2D + 2 * T2D * CF_ROWS);
}
inline size_t gptq2d_row_flush_smem(int band) {
    return sizeof(float) * ((size_t)band * T2D * UHS_PITCH + 2 * T2D * RF_COLS);
}

// ---------------------------------------------------------------------------------------
// Column flush of band [S0, S1] into the tiles of stages >= T0: for column strip J the band's
// rows are [lo, hi] = [max(0, S0 - J), min(MT - 1, S1 - J)], and every row p of the strip in
// a tile row I >= T0 - J gets
//   Cacc[p, J] += sum_k U_G[k, p] E[k, J],  k over the band rows.
// One item: 128 rows x 32 columns, 4 x 4 outputs per thread. The band's errors stay in shared
// memory; U_G streams through in 32-row chunks, double-buffered.
// ---------------------------------------------------------------------------------------
__device__ void col_flush_item(const Gptq2dArgs &a, int S0, int S1, int T0, int J, int chunk,
                               float *sm) {
    const int lo = max(0, S0 - J), hi = min(a.MT - 1, S1 - J);
    if (lo > hi) return;
    const long long p0 = (long long)max(hi + 1, T0 - J) * T2D + (long long)chunk * CF_ROWS;
    if (p0 >= a.Mp) return;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const long long c0 = (long long)J * T2D, k0 = (long long)lo * T2D;
    const int nk = hi - lo + 1;
    float *Bs = sm;                              // nk*32 x 32: E[k, q]
    float *As = sm + nk * T2D * T2D;             // 2 x 32 x 128: U_G[k, p]
    for (int c = tid; c < nk * T2D * 8; c += FLUSH_THREADS) {
        const int k = c >> 3, q = (c & 7) * 4;
        cp_async16(Bs + k * T2D + q, a.E + (k0 + k) * a.Np + c0 + q);
    }
    auto load_a = [&](int kt, int buf) {
        float *dst = As + buf * T2D * CF_ROWS;
        for (int c = tid; c < T2D * CF_ROWS / 4; c += FLUSH_THREADS) {
            const int k = c >> 5, q = (c & 31) * 4;
            const bool ok = p0 + q < a.Mp;
            const float *src = a.UG + (k0 + kt * T2D + k) * a.Mp + (ok ? p0 + q : 0);
            cp_async16_or_zero(dst + k * CF_ROWS + q, src, ok);
        }
    };
    load_a(0, 0);
    cp_async_commit();
    const int rg = lane >> 3, cg = lane & 7;
    const int row = w * 16 + rg * 4, col = cg * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int kt = 0; kt < nk; ++kt) {
        if (kt + 1 < nk) {
            load_a(kt + 1, (kt + 1) & 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const float *A = As + (kt & 1) * T2D * CF_ROWS;
        const float *B = Bs + kt * T2D * T2D;
#pragma unroll 8
        for (int k = 0; k < T2D; ++k) {
            const float4 av = *reinterpret_cast<const float4 *>(A + k * CF_ROWS + row);
            const float4 bv = *reinterpret_cast<const float4 *>(B + k * T2D + col);
            const float ar[4] = {av.x, av.y, av.z, av.w}, br[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] += ar[i] * br[j];
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const long long p = p0 + row + i;
        if (p < a.Mp) {
            float4 *dst = reinterpret_cast<float4 *>(a.Cacc + p * a.Np + c0 + col);
            float4 v = *dst;
            v.x += acc[i][0]; v.y += acc[i][1]; v.z += acc[i][2]; v.w += acc[i][3];
            *dst = v;
        }
    }
}

// ---------------------------------------------------------------------------------------
// Row flush of band [S0, S1] into the tiles of stages >= T0: for row strip I the band's
// columns are [lo, hi] = [max(0, S0 - I), min(NT - 1, S1 - I)], and every column q of the
// strip in a tile column J >= T0 - I gets
//   Xw[I, q] -= sum_k F[I, k] U_H[k, q],  k over the band columns.
// One item: 32 rows x 256 columns, 4 x 8 outputs per thread. The band's column buffer values
// stay in shared memory (transposed); U_H streams through in 32-row chunks, double-buffered.
// ---------------------------------------------------------------------------------------
__device__ void row_flush_item(const Gptq2dArgs &a, int S0, int S1, int T0, int I, int chunk,
                               float *sm) {
    const int lo = max(0, S0 - I), hi = min(a.NT - 1, S1 - I);
    if (lo > hi) return;
    const long long q0 = (long long)max(hi + 1, T0 - I) * T2D + (long long)chunk * RF_COLS;
    if (q0 >= a.Np) return;
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const long long r0 = (long long)I * T2D, k0 = (long long)lo * T2D;
    const int nk = hi - lo + 1, K = nk * T2D;
    float *Ft = sm;                                  // K x 36: F[r, k] stored at Ft[k][r]
    float *Bs = sm + nk * T2D * UHS_PITCH;           // 2 x 32 x 256: U_H[k, q]
    auto load_b = [&](int kt, int buf) {
        float *dst = Bs + buf * T2D * RF_COLS;
        for (int c = tid; c < T2D * RF_COLS / 4; c += FLUSH_THREADS) {
            const int k = c >> 6, q = (c & 63) * 4;
            const bool ok = q0 + q < a.Np;
            const float *src = a.UH + (k0 + kt * T2D + k) * a.Np + (ok ? q0 + q : 0);
            cp_async16_or_zero(dst + k * RF_COLS + q, src, ok);
        }
    };
    load_b(0, 0);
    cp_async_commit();
    for (int idx = tid; idx < T2D * K; idx += FLUSH_THREADS) {
        const int r = idx / K, k = idx - r * K;
        Ft[k * UHS_PITCH + r] = a.F[(r0 + r) * a.Np + k0 + k];
    }
    const int rg = lane >> 2, cg = lane & 3;
    const int row = rg * 4, col = w * 32 + cg * 8;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
    for (int kt = 0; kt < nk; ++kt) {
        if (kt + 1 < nk) {
            load_b(kt + 1, (kt + 1) & 1);
            cp_async_commit();
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();
        const float *B = Bs + (kt & 1) * T2D * RF_COLS;
        const float *A = Ft + kt * T2D * UHS_PITCH;
#pragma unroll 4
        for (int k = 0; k < T2D; ++k) {
            const float4 fv = *reinterpret_cast<const float4 *>(A + k * UHS_PITCH + row);
            const float4 b0 = *reinterpret_cast<const float4 *>(B + k * RF_COLS + col);
            const float4 b1 = *reinterpret_cast<const float4 *>(B + k * RF_COLS + col + 4);
            const float fr[4] = {fv.x, fv.y, fv.z, fv.w};
            const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[i][j] += fr[i] * br[j];
        }
        __syncthreads();
    }
    const long long q = q0 + col;
    if (q < a.Np) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 *dst = reinterpret_cast<float4 *>(a.Xw + (r0 + row + i) * a.Np + q);
            float4 v0 = dst[0], v1 = dst[1];
            v0.x -= acc[i][0]; v0.y -= acc[i][1]; v0.z -= acc[i][2]; v0.w -= acc[i][3];
            v1.x -= acc[i][4]; v1.y -= acc[i][5]; v1.z -= acc[i][6]; v1.w -= acc[i][7];
            dst[0] = v0;
            dst[1] = v1;
        }
    }
}

// The flush of one band into every later stage (T0 = S1 + 1), as two full grids: column items
// (NT x ceil(Mp / 128)) and row items (MT x ceil(Np / 256)).
__global__ __launch_bounds__(FLUSH_THREADS) void gptq2d_col_flush_kernel(Gptq2dArgs a, int S0, int S1) {
    pdl_launch_next();
    pdl_wait_prev();
    extern __shared__ __align__(16) float sm[];
    col_flush_item(a, S0, S1, S1 + 1, blockIdx.x, blockIdx.y, sm);
}
__global__ __launch_bounds__(FLUSH_THREADS) void gptq2d_row_flush_kernel(Gptq2dArgs a, int S0, int S1) {
    pdl_launch_next();
    pdl_wait_prev();
    extern __shared__ __align__(16) float sm[];
    row_flush_item(a, S0, S1, S1 + 1, blockIdx.x, blockIdx.y, sm);
}

// Xw <- X on the real entries, zero on the padding; Cacc <- 0.
__global__ void gptq2d_init_kernel(const float *X, int m, int n, float *Xw, float *Cacc,
                                   long long Mp, long long Np) {
    const long long total = Mp * Np;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long p = i / Np, q = i - p * Np;
        Xw[i] = (p < m && q < n) ? X[p * n + q] : 0.f;
        Cacc[i] = 0.f;
    }
}

// Rows [d0, dp) of a dp x dp factor (ld dp): identity rows for the padding.
__global__ void gptq2d_pad_identity_kernel(float *U, long long d0, long long dp) {
    const long long total = (dp - d0) * dp;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long r = d0 + i / dp, c = i % dp;
        U[r * dp + c] = r == c ? 1.f : 0.f;
    }
}

template <typename... KArgs, typename... Args>
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, int threads, size_t smem,
                      cudaStream_t s, Args... args) {
    return launch_kernel(kernel, grid, dim3(threads), smem, s, true, args...);
}

// Side stream on which U_G is factored while U_H is factored on the caller's stream (one per
// device, created on first use; `mu` serialises the fork / join of concurrent calls).
struct Gptq2dSide {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex mu;
    bool ready = false;
};

inline Gptq2dSide *gptq2d_side() {
    static Gptq2dSide sd[64];
    static std::mutex init_mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(init_mu);
    Gptq2dSide &g = sd[dev];
    if (!g.ready) {
        bool ok = cudaStreamCreateWithFlags(&g.stream, cudaStreamNonBlocking) == cudaSuccess &&
                  cudaEventCreateWithFlags(&g.fork, cudaEventDisableTiming) == cudaSuccess &&
                  cudaEventCreateWithFlags(&g.join, cudaEventDisableTiming) == cudaSuccess;
        if (!ok) return nullptr;
        g.ready = true;
    }
    return &g;
}

inline int gptq2d_band() {
    const char *e = std::getenv("GPTQ_2D_BAND");
    int w = e ? std::atoi(e) : T2D_BAND_DEFAULT;
    return w < 1 ? 1 : (w > T2D_BAND_MAX ? T2D_BAND_MAX : w);
}

// The wavefront: stages in bands of W tile anti-diagonals, a flush after every band that
// has a successor.
// The wavefront: tile anti-diagonals in bands of W; after each band that has a successor, its
// flush into all later tiles.
inline int gptq2d_sweep(Gptq2dArgs a, cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_2D);
    const int W = gptq2d_band();
    const int Smax = a.MT + a.NT - 2;
    const size_t smem = gptq2d_sweep_smem(W);
    const size_t smem_c = gptq2d_col_flush_smem(W), smem_r = gptq2d_row_flush_smem(W);
    if (cudaFuncSetAttribute(gptq2d_sweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess ||
        cudaFuncSetAttribute(gptq2d_col_flush_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_c) != cudaSuccess ||
        cudaFuncSetAttribute(gptq2d_row_flush_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem_r) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    for (int S0 = 0; S0 <= Smax; S0 += W) {
        const int S1 = std::min(S0 + W - 1, Smax);
        for (int S = S0; S <= S1; ++S) {
            const int tiles = std::min(S, a.MT - 1) - std::max(0, S - a.NT + 1) + 1;
            if (int st = launch_pdl(gptq2d_sweep_kernel, dim3(tiles), T2D_THREADS, smem, s, a, S, S0))
                return st;
        }
        if (S1 < Smax) {
            if (int st = launch_pdl(gptq2d_col_flush_kernel, dim3(a.NT, ceil_div(a.Mp, CF_ROWS)),
                                    FLUSH_THREADS, smem_c, s, a, S0, S1))
                return st;
            if (int st = launch_pdl(gptq2d_row_flush_kernel, dim3(a.MT, ceil_div(a.Np, RF_COLS)),
                                    FLUSH_THREADS, smem_r, s, a, S0, S1))
                return st;
        }
    }
    return GPTQ_OK;
}

}  // namespace gptq
