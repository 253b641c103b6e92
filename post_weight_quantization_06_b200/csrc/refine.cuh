// OLrC + Bid-Up refinement of an intrinsic-LoRA layer.
//
// GPTQ-intrinsic LoRA summary, section 4 ("Refinement by Bid-Up"): OLrC, the best low-rank
// L, R for the fixed quantized Q, alternates with Bid-Up, coordinate-wise updates of Q on
// its fixed grid for fixed L, R; each minimises the reconstruction error over its own
// variables, so the error never increases. In this library's orientation (W m x n, one
// neuron per row; dequantized weight Qhat + R^T L^T; G = X^T X, H = 2 G):
//   OLrC    E = W - Qhat; P = top-r eigenvectors of E H E^T (m x m); R = P^T, L = E^T P
//           (X (L R) is then the rank-r truncation of X E^T);
//   Bid-Up  D = E - P (P^T E), g = D H; for j = 0 .. n-1 (all rows at once): the new code
//           is clip(rint(c + g_j / (H_jj s)), 0, maxq), the grid point nearest the 1-D
//           optimum of that coordinate; qhat_j moves by delta = s (c_new - c), d_j by
//           -delta, and g by -delta H[j, :].
// Bid-Up's structure is the GPTQ sweep's (sequential coordinates, independent rows, a
// rank-1 feedback through the upper rows of a fixed n x n matrix), so it runs the same way:
// 128-column blocks with the block of H in shared memory and the rows in parallel, then a
// lazy GEMM that applies the block's changes to the later columns' gradients.
#pragma once

#include "common.cuh"
#include "gemm_tc.cuh"
#include "il.cuh"

namespace gptq {

// Packed codes (LSB-first bit stream per row, ldw 32-bit words per row) <-> one byte per code.
__global__ void refine_unpack_kernel(const uint32_t *codes, long long ldw, int m, int n,
                                     int bits, uint8_t *out, long long ldo) {
    const long long total = (long long)m * n;
    const uint32_t mask = (1u << bits) - 1u;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int o = (int)(idx / n), j = (int)(idx % n);
        const long long p = (long long)j * bits;
        const uint32_t *row = codes + (long long)o * ldw;
        const int w = (int)(p >> 5), off = (int)(p & 31);
        uint32_t v = row[w] >> off;
        if (off + bits > 32) v |= row[w + 1] << (32 - off);
        out[(long long)o * ldo + j] = (uint8_t)(v & mask);
    }
}

__global__ void refine_pack_kernel(const uint8_t *in, long long ldi, int m, int n, int bits,
                                   uint32_t *codes, long long ldw) {
    const int words = n * bits / 32;
    const long long total = (long long)m * words;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int o = (int)(idx / words), w = (int)(idx % words);
        const int bit0 = 32 * w;
        const int cfirst = bit0 / bits, clast = min(n - 1, (bit0 + 31) / bits);
        uint32_t word = 0;
        for (int c = cfirst; c <= clast; ++c) {
            const int pos = c * bits - bit0;
            const uint32_t code = in[(long long)o * ldi + c];
            word |= pos >= 0 ? (code << pos) : (code >> (-pos));
        }
        codes[(long long)o * ldw + w] = word;
    }
}

// E = W - Qhat, Qhat[o, j] = s[o, g] (c[o, j] - z[o, g]), g = j / gs.
template <typename TW>
__global__ void refine_error_kernel(const TW *W, int m, int n, const uint8_t *c, const float *scales,
                                    const uint8_t *zeros, int G, int gs, float *E) {
    const long long total = (long long)m * n;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int o = (int)(idx / n), j = (int)(idx % n);
        const int g = j / gs;
        const float s = scales[(long long)o * G + g], z = (float)zeros[(long long)o * G + g];
        E[idx] = to_f32(W[idx]) - s * ((float)c[idx] - z);
    }
}

// R = P^T (P m x r, R r x m).
__global__ void refine_transpose_kernel(const float *P, int m, int r, float *R) {
    const long long total = (long long)m * r;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(idx / m), o = (int)(idx % m);
        R[idx] = P[(long long)o * r + t];
    }
}

// rowloss[o] = sum_j D[o, j] g[o, j] (= d_o H d_o^T), one warp per row, fp64 sums.
__global__ void refine_rowdot_kernel(const float *D, const float *g, int m, int n, double *rowloss) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= m) return;
    double acc = 0.0;
    for (int j = lane; j < n; j += 32)
        acc += (double)D[(long long)warp * n + j] * (double)g[(long long)warp * n + j];
    acc = warp_sum_d(acc);
    if (lane == 0) rowloss[warp] = acc;
}

// out = sum_o rowloss[o] / 2 (the reconstruction error with G = H / 2), fixed order.
__global__ void refine_total_kernel(const double *rowloss, int m, double *out) {
    __shared__ double part[32];
    double acc = 0.0;
    for (int i = threadIdx.x; i < m; i += blockDim.x) acc += rowloss[i];
    acc = warp_sum_d(acc);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
        v = warp_sum_d(v);
        if (threadIdx.x == 0) *out = 0.5 * v;
    }
}

struct BidupArgs {
    const float *H;     // n x n (undamped 2 X^T X), row-major
    long long ldh;
    float *g;           // m x n gradients d H; the block's columns are read
    long long ldg;
    uint8_t *codes;     // m x n, one byte per code, updated in place
    long long ldc;
    const float *scales;
    int G, gs;
    float *err;         // m x B: change of qhat per column of the block (lazy update input)
    long long lde;
    double *rowloss;    // per row d H d^T, advanced by every accepted step
    int m, n, j0, bits;
};

// One CTA = 8 warps, one warp = ROWS rows, lane l owns columns l, l+32, ... of the block.
// Per column t: the owner lane's gradient, code and scale are broadcast by shuffle, every
// lane evaluates the decision for its rows (the same on all lanes), and the lanes apply
// -delta H[t, col] to the gradients of the block columns after t.
template <int NSLOT, int ROWS>
__global__ __launch_bounds__(256) void bidup_block_kernel(BidupArgs a) {
    constexpr int B = 32 * NSLOT;
    extern __shared__ float bsm[];
    float *Hs = bsm;          // B x B block of H
    float *hinv = Hs + B * B; // 1 / H_tt, 0 where H_tt <= 0 (coordinate left alone)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int j0 = a.j0;
    for (int base = tid; base < B * B; base += 8 * blockDim.x) {
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = base + u * blockDim.x, t = idx / B, c = idx % B;
            v[u] = (idx < B * B && j0 + t < a.n && j0 + c < a.n)
                       ? a.H[(long long)(j0 + t) * a.ldh + j0 + c] : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int idx = base + u * blockDim.x;
            if (idx < B * B) Hs[idx] = v[u];
        }
    }
    __syncthreads();
    for (int t = tid; t < B; t += blockDim.x) {
        const float h = Hs[t * B + t];
        hinv[t] = h > 0.f ? 1.f / h : 0.f;
    }
    __syncthreads();

    const float fmaxq = (float)((1 << a.bits) - 1);
    const int row0 = (blockIdx.x * nwarps + warp) * ROWS;
    float g[ROWS][NSLOT], cv[ROWS][NSLOT], sv[ROWS][NSLOT], dv[ROWS][NSLOT];
    float dl[ROWS];
    bool rv[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const int row = row0 + r;
        rv[r] = row < a.m;
        dl[r] = 0.f;
#pragma unroll
        for (int q = 0; q < NSLOT; ++q) {
            const int col = j0 + 32 * q + lane;
            const bool ok = rv[r] && col < a.n;
            g[r][q] = ok ? a.g[(long long)row * a.ldg + col] : 0.f;
            cv[r][q] = ok ? (float)a.codes[(long long)row * a.ldc + col] : 0.f;
            sv[r][q] = ok ? a.scales[(long long)row * a.G + col / a.gs] : 1.f;
            dv[r][q] = 0.f;
        }
    }
#pragma unroll
    for (int q = 0; q < NSLOT; ++q) {
#pragma unroll 2
        for (int o = 0; o < 32; ++o) {
            const int t = 32 * q + o;
            if (j0 + t >= a.n) break;
            const float ih = hinv[t], htt = Hs[t * B + t];
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const float gt = __shfl_sync(0xffffffffu, g[r][q], o);
                const float ct = __shfl_sync(0xffffffffu, cv[r][q], o);
                const float st = __shfl_sync(0xffffffffu, sv[r][q], o);
                const float v = ct + gt * ih / st;
                const float cn = ih > 0.f ? fminf(fmaxf(rintf(v), 0.f), fmaxq) : ct;
                const float delta = st * (cn - ct);
                dl[r] = fmaf(delta, fmaf(delta, htt, -2.f * gt), dl[r]);
                if (lane == o) {
                    cv[r][q] = cn;
                    dv[r][q] = delta;
                }
#pragma unroll
                for (int q2 = q; q2 < NSLOT; ++q2) {
                    const int col = 32 * q2 + lane;
                    if (q2 > q || lane > o) g[r][q2] = fmaf(-delta, Hs[t * B + col], g[r][q2]);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const int row = row0 + r;
        if (!rv[r]) continue;
#pragma unroll
        for (int q = 0; q < NSLOT; ++q) {
            const int col = j0 + 32 * q + lane;
            a.err[(long long)row * a.lde + 32 * q + lane] = dv[r][q];
            if (col < a.n) a.codes[(long long)row * a.ldc + col] = (uint8_t)cv[r][q];
        }
        if (lane == 0) a.rowloss[row] += (double)dl[r];
    }
}

constexpr int BIDUP_B = 128, BIDUP_ROWS = 2, BIDUP_THREADS = 256;

// Workspace of the refinement (m x n layer, rank r).
struct RefineWs {
    float *E, *Gm, *D, *Bm, *P, *Z, *Err;
    uint8_t *c8;
    double *rowloss;
    ILWork il;
};

// One Bid-Up pass over all columns: g = D H on entry (in Gm), codes updated in c8, the
// per-row loss advanced from its value on entry.
inline int bidup_pass(const float *H, int m, int n, int bits, int gs, const float *scales,
                      RefineWs &w, cudaStream_t s) {
    constexpr int B = BIDUP_B;
    const size_t smem = sizeof(float) * (B * B + B);
    GPTQ_SMEM_LIMIT((bidup_block_kernel<B / 32, BIDUP_ROWS>), smem);
    const int G = n / gs;
    const int rows_per_cta = (BIDUP_THREADS / 32) * BIDUP_ROWS;
    for (int j0 = 0; j0 < n; j0 += B) {
        BidupArgs a;
        a.H = H; a.ldh = n;
        a.g = w.Gm; a.ldg = n;
        a.codes = w.c8; a.ldc = n;
        a.scales = scales; a.G = G; a.gs = gs;
        a.err = w.Err; a.lde = B;
        a.rowloss = w.rowloss;
        a.m = m; a.n = n; a.j0 = j0; a.bits = bits;
        bidup_block_kernel<B / 32, BIDUP_ROWS>
            <<<ceil_div(m, rows_per_cta), BIDUP_THREADS, smem, s>>>(a);
        if (int st = launch_status()) return st;
        const int j1 = j0 + B;
        if (j1 < n) {
            // g[:, j1:] -= Err (m x B) H[j0:j1, j1:]
            auto p = gemm_args<float, float>(m, n - j1, B, w.Err, B, 0, H + (long long)j0 * n + j1,
                                             n, 0, w.Gm + j1, n, -1.f, 1.f);
            if (int st = gemm_f32(p, s)) return st;
        }
    }
    return GPTQ_OK;
}

// The refinement loop; codes8 holds the pass's codes (one byte each) on entry and the
// refined ones on exit; loss_hist receives 2 iters values (after each OLrC and Bid-Up).
template <typename TW>
inline int il_refine(const TW *W, int m, int n, const float *H, int r, int bits, int gs,
                     int iters, const float *scales, const uint8_t *zeros, float *L, float *R,
                     double *loss_hist, RefineWs &w, cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_REFINE);
    const int G = n / gs;
    const long long mn = (long long)m * n;
    const int blocks = (int)std::min<long long>((mn + 255) / 256, 148LL * 8);
    for (int it = 0; it < iters; ++it) {
        // ---- OLrC: E = W - Qhat, Bm = E H E^T, P = top-r eigenvectors, L = E^T P, R = P^T
        refine_error_kernel<TW><<<blocks, 256, 0, s>>>(W, m, n, w.c8, scales, zeros, G, gs, w.E);
        GPTQ_CHECK_LAUNCH();
        if (r > 0) {
            if (int st = gemm_f32(gemm_args<float, float>(m, n, n, w.E, n, 0, H, n, 0, w.Gm, n,
                                                          1.f, 0.f), s)) return st;
            if (int st = gemm_f32(gemm_args<float, float>(m, m, n, w.Gm, n, 0, w.E, n, 1, w.Bm, m,
                                                          1.f, 0.f), s)) return st;
            if (int st = il_top_eigvecs(w.Bm, m, m, r, w.P, w.il, s, false)) return st;
            if (int st = gemm_f32(gemm_args<float, float>(n, r, m, w.E, n, 1, w.P, r, 0, L, r,
                                                          1.f, 0.f), s)) return st;
            refine_transpose_kernel<<<blocks, 256, 0, s>>>(w.P, m, r, R);
            GPTQ_CHECK_LAUNCH();
            // ---- D = E - P (P^T E)
            if (int st = gemm_f32(gemm_args<float, float>(r, n, m, w.P, r, 1, w.E, n, 0, w.Z, n,
                                                          1.f, 0.f), s)) return st;
            if (cudaMemcpyAsync(w.D, w.E, sizeof(float) * mn, cudaMemcpyDeviceToDevice, s) !=
                cudaSuccess)
                return GPTQ_ERR_CUDA;
            if (int st = gemm_f32(gemm_args<float, float>(m, n, r, w.P, r, 0, w.Z, n, 0, w.D, n,
                                                          -1.f, 1.f), s)) return st;
        } else if (cudaMemcpyAsync(w.D, w.E, sizeof(float) * mn, cudaMemcpyDeviceToDevice, s) !=
                   cudaSuccess) {
            return GPTQ_ERR_CUDA;
        }
        // ---- g = D H and the loss after OLrC
        if (int st = gemm_f32(gemm_args<float, float>(m, n, n, w.D, n, 0, H, n, 0, w.Gm, n, 1.f,
                                                      0.f), s)) return st;
        refine_rowdot_kernel<<<ceil_div(m, 8), 256, 0, s>>>(w.D, w.Gm, m, n, w.rowloss);
        GPTQ_CHECK_LAUNCH();
        refine_total_kernel<<<1, 1024, 0, s>>>(w.rowloss, m, loss_hist + 2 * it);
        GPTQ_CHECK_LAUNCH();
        // ---- Bid-Up and the loss after it
        if (int st = bidup_pass(H, m, n, bits, gs, scales, w, s)) return st;
        refine_total_kernel<<<1, 1024, 0, s>>>(w.rowloss, m, loss_hist + 2 * it + 1);
        GPTQ_CHECK_LAUNCH();
    }
    return GPTQ_OK;
}

// ---------------------------------------------------------------------------------------
// Low-precision storage of the low-rank factors (GPTQ-intrinsic LoRA summary, "Main
// results": 4-bit L and 8-bit R are often lossless): round-to-nearest onto the pass's
// per-group min-max grid, each factor stored one neuron per row. A(row, col) =
// A[row * rs + col * cs] (L^T: rs = 1, cs = r; R^T: rs = 1, cs = m). One warp per row:
// group ranges by warp reduction, the grid by the sweep's own rule (grid_from_range), then
// the packed words, each lane recomputing the codes of the words it writes.
// ---------------------------------------------------------------------------------------
__global__ void rtn_rows_kernel(const float *A, long long rs, long long cs, int rows, int cols,
                                int bits, int gs, uint32_t *codes, long long ldw, float *scales,
                                uint8_t *zeros, int G) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
    if (warp >= rows) return;
    const float fmaxq = (float)((1 << bits) - 1);
    const float *a = A + (long long)warp * rs;
    for (int g = 0; g < G; ++g) {
        float mn = INFINITY, mx = -INFINITY;
        for (int c = g * gs + lane; c < min(cols, (g + 1) * gs); c += 32) {
            const float x = a[(long long)c * cs];
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
        }
        mn = warp_min(mn);
        mx = warp_max(mx);
        float s, is, z;
        grid_from_range(mn, mx, fmaxq, s, is, z);
        if (lane == 0) {
            scales[(long long)warp * G + g] = s;
            zeros[(long long)warp * G + g] = (uint8_t)z;
        }
    }
    __syncwarp();
    const int words = cols * bits / 32;
    for (int w = lane; w < words; w += 32) {
        const int bit0 = 32 * w;
        const int cfirst = bit0 / bits, clast = min(cols - 1, (bit0 + 31) / bits);
        uint32_t word = 0;
        for (int c = cfirst; c <= clast; ++c) {
            const int g = c / gs;
            const float s = scales[(long long)warp * G + g];
            const float z = (float)zeros[(long long)warp * G + g];
            const float v = fmaf(a[(long long)c * cs], __frcp_rn(s), z);
            const uint32_t code = (uint32_t)fminf(fmaxf(rintf(v), 0.f), fmaxq);
            const int pos = c * bits - bit0;
            word |= pos >= 0 ? (code << pos) : (code >> (-pos));
        }
        codes[(long long)warp * ldw + w] = word;
    }
}

}  // namespace gptq
