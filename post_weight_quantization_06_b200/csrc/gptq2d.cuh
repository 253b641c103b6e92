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
// band's errors are flushed into all later tiles at once (the banded product of the blocked
// algorithm):
//   Cacc[p, J] += U_G[band rows of J, p]^T E[band rows, J]   (column flush)
//   Xw[I, q]  -= F[I, band cols of I] U_H[band cols, q]       (row flush)
// where F is the final column buffer (C after the entry's own error) and Xw = X minus all
// flushed row pushes. Padded rows / columns (m, n not multiples of 32) carry zero input and
// identity factors; feedback only flows down and right, so they never reach a real entry.
#pragma once

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

// Programmatic dependent launch: every kernel of the wavefront lets the next one start at
// once (its independent prologue overlaps this kernel) and waits for the previous kernel's
// completion before it touches anything that kernel wrote.
__device__ __forceinline__ void pdl_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

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
// dynamic shared memory of the sweep: 9 fixed tiles (Cs, Xs, UGd, UHs with its reciprocals
// (two tiles), Es, Fs, Zs) and two operand tiles per pulled tile
inline size_t gptq2d_sweep_smem(int band) { return sizeof(float) * T2D_TILE * (9 + 4 * (band - 1)); }

// Physical register p of a rotated row holds slot (base + p) % 32; shifting the array down by
// R after R steps keeps the slot of the current step at index 0 .. R-1.
template <int R>
__device__ __forceinline__ void rotate_down(float (&x)[T2D]) {
    float t[R];
#pragma unroll
    for (int i = 0; i < R; ++i) t[i] = x[i];
#pragma unroll
    for (int i = 0; i < T2D - R; ++i) x[i] = x[i + R];
#pragma unroll
    for (int i = 0; i < R; ++i) x[T2D - R + i] = t[i];
}

// ---------------------------------------------------------------------------------------
// Tile sweep of stage S (tiles with I + J = S), band starting at stage S0. One CTA per tile.
// All operands are copied to shared memory at once; the four warps add the band's earlier
// tiles (pulls), then warp 0 sweeps the tile's 63 anti-diagonals. The error is formed with
// the reciprocals of the two diagonal entries (within a few ulp of the quotient).
// ---------------------------------------------------------------------------------------
constexpr int T2D_UNROLL = 8;

__global__ __launch_bounds__(T2D_THREADS) void gptq2d_sweep_kernel(Gptq2dArgs a, int S, int S0) {
    extern __shared__ __align__(16) float sm[];
    float *Cs = sm, *Xs = sm + T2D_TILE, *UGd = sm + 2 * T2D_TILE;
    // U_H[J, J] with row b shifted left by b: UHs[b][k] = U_H[b, b + k] (zero past the tile),
    // pitch 36 so that the lanes' 16-byte row reads fall in distinct banks
    float *UHs = sm + 3 * T2D_TILE;
    float *ruh = UHs + T2D * UHS_PITCH;                 // 1 / U_H[b, b]
    float *Es = sm + 5 * T2D_TILE, *Fs = sm + 6 * T2D_TILE;
    int *Zs = reinterpret_cast<int *>(sm + 7 * T2D_TILE);
    float *P = sm + 9 * T2D_TILE;                       // pulled operand pairs

    const int tid = threadIdx.x;
    const int I = max(0, S - a.NT + 1) + blockIdx.x;
    const int J = S - I;
    const long long r0g = (long long)I * T2D, c0g = (long long)J * T2D;
    const int i_lo = max(0, S0 - J), j_lo = max(0, S0 - I);
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
        UHs[r * UHS_PITCH + k] = r + k < T2D ? a.UH[(c0g + r) * a.Np + c0g + r + k] : 0.f;
        if (k == 0) ruh[r] = 1.f / a.UH[(c0g + r) * a.Np + c0g + r];
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
        const int l = tx;
        float xw[T2D], cc[T2D], ugc[T2D];
#pragma unroll
        for (int p = 0; p < T2D; ++p) {
            const int col = (p - l) & 31;
            xw[p] = Xs[l * T2D + col];
            cc[p] = Cs[l * T2D + col];
        }
        ugc[0] = 0.f;
#pragma unroll
        for (int d = 1; d < T2D; ++d) ugc[d] = l >= d ? UGd[(l - d) * T2D + l] : 0.f;   // U_G[l-d, l]
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
                const float *uhrow = UHs + bc * UHS_PITCH;
                float uh[T2D];
#pragma unroll
                for (int k4 = 0; k4 < T2D; k4 += 4) {
                    const float4 t4 = *reinterpret_cast<const float4 *>(uhrow + k4);
                    uh[k4] = t4.x; uh[k4 + 1] = t4.y; uh[k4 + 2] = t4.z; uh[k4 + 3] = t4.w;
                }
                const float rinv = rug * ruh[bc];
                const float v = xw[u] - cc[u] * uh[0];
                const float z = rintf(v);
                const float e = act ? (v - z) * rinv : 0.f;
                const float cf = act ? cc[u] + ugd * e : 0.f;
                if (act) {
                    bad |= !isfinite(v);
                    Zs[l * T2D + b] = __float2int_rn(z);
                    Es[l * T2D + b] = e;
                    Fs[l * T2D + b] = cf;
                }
                // error down the column: lane l - d decided column b + d, held in slot u + d
#pragma unroll
                for (int d = 1; d < T2D; ++d) {
                    const float ed = __shfl_up_sync(0xffffffffu, e, d);
                    cc[(u + d) & 31] += ugc[d] * ed;
                }
                // final column buffer value along the own row
#pragma unroll
                for (int k = 1; k < T2D; ++k) xw[(u + k) & 31] -= cf * uh[k];
            }
            rotate_down<T2D_UNROLL>(xw);
            rotate_down<T2D_UNROLL>(cc);
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

// ---------------------------------------------------------------------------------------
// Column flush of band [S0, S1]: for each column strip J, the band's rows of J are
// [lo, hi] = [max(0, S0 - J), min(MT - 1, S1 - J)]; every later row p of the strip gets
//   Cacc[p, J] += sum_k U_G[k, p] E[k, J],  k over the band rows.
// Grid (NT, ceil(Mp / 64)); CTA: 64 rows x 32 columns, 16 outputs per thread.
// ---------------------------------------------------------------------------------------
__global__ __launch_bounds__(T2D_THREADS) void gptq2d_col_flush_kernel(Gptq2dArgs a, int S0, int S1) {
    pdl_launch_next();
    pdl_wait_prev();
    __shared__ __align__(16) float As[T2D][64];   // U_G[k, p]
    __shared__ __align__(16) float Bs[T2D][T2D];  // E[k, q]
    const int J = blockIdx.x;
    const int lo = max(0, S0 - J), hi = min(a.MT - 1, S1 - J);
    if (lo > hi) return;
    const long long p0 = (long long)(hi + 1) * T2D + (long long)blockIdx.y * 64;
    if (p0 >= a.Mp) return;
    const int tid = threadIdx.x, tx = tid & 31, ty = tid >> 5;
    const long long c0 = (long long)J * T2D;
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    for (int kt = lo; kt <= hi; ++kt) {
        const long long k0 = (long long)kt * T2D;
        __syncthreads();
        for (int t = tid; t < T2D * 64; t += T2D_THREADS) {
            const int k = t >> 6, c = t & 63;
            As[k][c] = p0 + c < a.Mp ? a.UG[(k0 + k) * a.Mp + p0 + c] : 0.f;
        }
        for (int t = tid; t < T2D * T2D; t += T2D_THREADS) {
            const int k = t >> 5, c = t & 31;
            Bs[k][c] = a.E[(k0 + k) * a.Np + c0 + c];
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < T2D; ++k) {
            const float b = Bs[k][tx];
            const float4 *ap = reinterpret_cast<const float4 *>(&As[k][ty * 16]);
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                const float4 av = ap[i4];
                acc[4 * i4 + 0] += av.x * b;
                acc[4 * i4 + 1] += av.y * b;
                acc[4 * i4 + 2] += av.z * b;
                acc[4 * i4 + 3] += av.w * b;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const long long p = p0 + ty * 16 + i;
        if (p < a.Mp) a.Cacc[p * a.Np + c0 + tx] += acc[i];
    }
}

// ---------------------------------------------------------------------------------------
// Row flush of band [S0, S1]: for each row strip I, the band's columns of I are
// [lo, hi] = [max(0, S0 - I), min(NT - 1, S1 - I)]; every later column q of the strip gets
//   Xw[I, q] -= sum_k F[I, k] U_H[k, q],  k over the band columns.
// Grid (MT, ceil(Np / 128)); CTA: 32 rows x 128 columns, 32 outputs per thread (a column).
// ---------------------------------------------------------------------------------------
__global__ __launch_bounds__(T2D_THREADS) void gptq2d_row_flush_kernel(Gptq2dArgs a, int S0, int S1) {
    pdl_launch_next();
    pdl_wait_prev();
    __shared__ __align__(16) float Ft[T2D][T2D + 4];  // F[p, k] stored transposed: Ft[k][p]
    __shared__ __align__(16) float Bs[T2D][128];      // U_H[k, q]
    const int I = blockIdx.x;
    const int lo = max(0, S0 - I), hi = min(a.NT - 1, S1 - I);
    if (lo > hi) return;
    const long long q0 = (long long)(hi + 1) * T2D + (long long)blockIdx.y * 128;
    if (q0 >= a.Np) return;
    const int tid = threadIdx.x;
    const long long r0 = (long long)I * T2D;
    float acc[T2D];
#pragma unroll
    for (int i = 0; i < T2D; ++i) acc[i] = 0.f;
    for (int kt = lo; kt <= hi; ++kt) {
        const long long k0 = (long long)kt * T2D;
        __syncthreads();
        for (int t = tid; t < T2D * T2D; t += T2D_THREADS) {
            const int r = t >> 5, k = t & 31;
            Ft[k][r] = a.F[(r0 + r) * a.Np + k0 + k];
        }
        for (int t = tid; t < T2D * 128; t += T2D_THREADS) {
            const int k = t >> 7, c = t & 127;
            Bs[k][c] = q0 + c < a.Np ? a.UH[(k0 + k) * a.Np + q0 + c] : 0.f;
        }
        __syncthreads();
#pragma unroll 2
        for (int k = 0; k < T2D; ++k) {
            const float b = Bs[k][tid];
            const float4 *fp = reinterpret_cast<const float4 *>(&Ft[k][0]);
#pragma unroll
            for (int i4 = 0; i4 < T2D / 4; ++i4) {
                const float4 f = fp[i4];
                acc[4 * i4 + 0] += f.x * b;
                acc[4 * i4 + 1] += f.y * b;
                acc[4 * i4 + 2] += f.z * b;
                acc[4 * i4 + 3] += f.w * b;
            }
        }
    }
    const long long q = q0 + tid;
    if (q < a.Np) {
#pragma unroll
        for (int i = 0; i < T2D; ++i) a.Xw[(r0 + i) * a.Np + q] -= acc[i];
    }
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
inline int launch_pdl(void (*kernel)(KArgs...), dim3 grid, size_t smem, cudaStream_t s,
                      Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(T2D_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, args...) != cudaSuccess) {
        launch_status();
        return GPTQ_ERR_CUDA;
    }
    return launch_status();
}

inline int gptq2d_band() {
    const char *e = std::getenv("GPTQ_2D_BAND");
    int w = e ? std::atoi(e) : T2D_BAND_DEFAULT;
    return w < 1 ? 1 : (w > T2D_BAND_MAX ? T2D_BAND_MAX : w);
}

// The wavefront: stages in bands of W tile anti-diagonals, a flush after every band that
// has a successor.
inline int gptq2d_sweep(Gptq2dArgs a, cudaStream_t s) {
    const int W = gptq2d_band();
    const int Smax = a.MT + a.NT - 2;
    const size_t smem = gptq2d_sweep_smem(W);
    if (cudaFuncSetAttribute(gptq2d_sweep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    for (int S0 = 0; S0 <= Smax; S0 += W) {
        const int S1 = S0 + W - 1 < Smax ? S0 + W - 1 : Smax;
        for (int S = S0; S <= S1; ++S) {
            const int tiles = (S < a.MT - 1 ? S : a.MT - 1) - (S - a.NT + 1 > 0 ? S - a.NT + 1 : 0) + 1;
            if (int st = launch_pdl(gptq2d_sweep_kernel, dim3(tiles), smem, s, a, S, S0)) return st;
        }
        if (S1 < Smax) {
            if (int st = launch_pdl(gptq2d_col_flush_kernel, dim3(a.NT, ceil_div(a.Mp, 64)), 0, s,
                                    a, S0, S1))
                return st;
            if (int st = launch_pdl(gptq2d_row_flush_kernel, dim3(a.MT, ceil_div(a.Np, 128)), 0, s,
                                    a, S0, S1))
                return st;
        }
    }
    return GPTQ_OK;
}

}  // namespace gptq
