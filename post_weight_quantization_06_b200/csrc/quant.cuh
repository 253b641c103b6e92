// The column sweep: per-group min-max grid, quantize/round/clamp, error feedback inside a
// panel of B columns, and the lazy trailing update once per panel.
//
// GPTQ (encyclopedia article), "Technical approach": columns are quantized one at a time
// and the remaining weights are corrected in closed form; groups carry their own scale.
// GPTQ-2D, section 2: errors of a block are flushed to the rest of the matrix with one
// matrix product (GPTQ's lazy block update).
#pragma once

#include "common.cuh"
#include "gemm_simt.cuh"
#include "gemm_tc.cuh"

namespace gptq {

// Wc[i, c] = W[i, c] for c < n, 0 for n <= c < N (the intrinsic-LoRA extra columns).
template <typename TW>
__global__ void init_work_kernel(const TW *W, long long m, int n, float *Wc, long long ldw, int N) {
    const long long total = m * (long long)N;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long row = idx / N;
        const int c = (int)(idx % N);
        float v = 0.f;
        if (c < n) {
            v = to_f32(W[row * n + c]);
            if (!isfinite(v)) report(GPTQ_ERR_NONFINITE, row * n + c);
        }
        Wc[row * ldw + c] = v;
    }
}

struct ColloopArgs {
    float *Wc;          // m x N working weights (row stride ldw)
    long long ldw;
    const float *U;     // n x N upper factor rows (row stride ldu)
    long long ldu;
    int m, n;           // rows, quantized columns
    int j0;             // first column of this panel
    int bits;
    int gs;             // group length (n when there is one group per row)
    uint32_t *codes;    // m x (n*bits/32)
    long long ldcodes;
    float *scales;      // m x G
    uint8_t *zeros;     // m x G
    int G;
    float *err;         // errors of this panel: m x B block at err (row stride lde), as the
    float *err_lo;      // tf32 pair hi = tf32(e) (err), lo = tf32(e - hi) (err_lo) that the
    long long lde;      // lazy update's tensor-core product takes without converting them
    double *loss;       // m or nullptr
};

// Grid of one group from its range: s = (xmax - xmin)/maxq, z = rint(-xmin/s) in [0, maxq].
__device__ __forceinline__ void grid_from_range(float mn, float mx, float fmaxq, float &s,
                                                float &is, float &z) {
    mn = fminf(mn, 0.f);
    mx = fmaxf(mx, 0.f);
    if (mx == mn) { mn = -1.f; mx = 1.f; }
    s = __fdiv_rn(mx - mn, fmaxq);
    is = __frcp_rn(s);
    z = fminf(fmaxf(rintf(__fdiv_rn(-mn, s)), 0.f), fmaxq);
}

// One CTA = 8 warps; one warp = ROWS rows; lane l owns columns l, l+32, ... of the panel.
// The panel's U block (B x B) and 1/U_jj sit in shared memory. Per column t: the owner
// lane's value is broadcast by shuffle, every lane evaluates the rounding of that column
// for its rows (the same value on all lanes), and each lane applies -e * U[t, col] to the
// columns it owns that come after t.
template <int NSLOT, int ROWS>
__global__ __launch_bounds__(256) void colloop_kernel(ColloopArgs a) {
    constexpr int B = 32 * NSLOT;
    extern __shared__ float sm[];
    float *Us = sm;
    float *invd = Us + B * B;
    uint8_t *cbuf = reinterpret_cast<uint8_t *>(invd + B);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int j0 = a.j0;
    // U block load: with 16-byte aligned rows all of it goes out at once as cp.async (the
    // weight rows below load meanwhile); otherwise eight plain loads in flight per thread
    const bool async_u = ((reinterpret_cast<uintptr_t>(a.U) | (uintptr_t)(a.ldu * 4)) & 15u) == 0;
    if (async_u) {
        for (int c = tid; c < B * B / 4; c += blockDim.x) {
            const int row = c / (B / 4), q4 = (c % (B / 4)) * 4;
            const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(Us + row * B + q4));
            const float *src = a.U + (long long)(j0 + row) * a.ldu + j0 + q4;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    } else {
        for (int base = tid; base < B * B; base += 8 * blockDim.x) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = base + u * blockDim.x;
                v[u] = idx < B * B ? a.U[(long long)(j0 + idx / B) * a.ldu + j0 + idx % B] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int idx = base + u * blockDim.x;
                if (idx < B * B) Us[idx] = v[u];
            }
        }
    }

    const int maxq = (1 << a.bits) - 1;
    const float fmaxq = (float)maxq;
    const int row0 = (blockIdx.x * nwarps + warp) * ROWS;
    float w[ROWS][NSLOT];
    float s[ROWS], is[ROWS], z[ROWS];
    bool rv[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const int row = row0 + r;
        rv[r] = row < a.m;
        s[r] = 1.f; is[r] = 1.f; z[r] = 0.f;
#pragma unroll
        for (int q = 0; q < NSLOT; ++q) {
            w[r][q] = rv[r] ? a.Wc[(long long)row * a.ldw + j0 + 32 * q + lane] : 0.f;
        }
    }
    if (async_u) asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    for (int t = tid; t < B; t += blockDim.x) invd[t] = 1.0f / Us[t * B + t];
    __syncthreads();
    const int gs = a.gs;
    const bool groups_in_panel = gs <= B;  // then B % gs == 0, so gs is a power of two
    const int gmask = groups_in_panel ? gs - 1 : 0;
    if (!groups_in_panel) {
        const int g = j0 / gs;
        if (j0 % gs == 0) {
            const int cend = min(j0 + gs, a.n);
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const int row = row0 + r;
                float mn = INFINITY, mx = -INFINITY;
                if (rv[r])
                    for (int c = j0 + lane; c < cend; c += 32) {
                        const float x = a.Wc[(long long)row * a.ldw + c];
                        mn = fminf(mn, x);
                        mx = fmaxf(mx, x);
                    }
                mn = warp_min(mn);
                mx = warp_max(mx);
                grid_from_range(mn, mx, fmaxq, s[r], is[r], z[r]);
                if (lane == 0 && rv[r]) {
                    a.scales[(long long)row * a.G + g] = s[r];
                    a.zeros[(long long)row * a.G + g] = (uint8_t)z[r];
                }
            }
        } else {
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const int row = row0 + r;
                if (rv[r]) {
                    s[r] = a.scales[(long long)row * a.G + g];
                    z[r] = (float)a.zeros[(long long)row * a.G + g];
                    is[r] = __frcp_rn(s[r]);
                }
            }
        }
    }

    // The panel's slots one after the other, the current one always in register slot 0: after
    // each slot the registers rotate down by one, so the loop over slots is a real loop whose
    // body (32 column steps, partly unrolled) is fetched once and reused NSLOT times.
    uint8_t *cb = cbuf + warp * ROWS * B;
    double lacc[ROWS];
#pragma unroll
    for (int r = 0; r < ROWS; ++r) lacc[r] = 0.0;
#pragma unroll 1
    for (int q = 0; q < NSLOT; ++q) {
        float cvc[ROWS], evc[ROWS];
#pragma unroll
        for (int r = 0; r < ROWS; ++r) { cvc[r] = 0.f; evc[r] = 0.f; }
#pragma unroll 4
        for (int o = 0; o < 32; ++o) {
            const int t = 32 * q + o;
            if (groups_in_panel && (t & gmask) == 0) {
                const int g = (j0 + t) / gs;
#pragma unroll
                for (int r = 0; r < ROWS; ++r) {
                    float mn = INFINITY, mx = -INFINITY;
#pragma unroll
                    for (int sl = 0; sl < NSLOT; ++sl) {
                        const int col = 32 * (q + sl) + lane;
                        if (q + sl < NSLOT && col >= t && col < t + gs) {
                            mn = fminf(mn, w[r][sl]);
                            mx = fmaxf(mx, w[r][sl]);
                        }
                    }
                    mn = warp_min(mn);
                    mx = warp_max(mx);
                    grid_from_range(mn, mx, fmaxq, s[r], is[r], z[r]);
                    if (lane == 0 && rv[r]) {
                        const int row = row0 + r;
                        a.scales[(long long)row * a.G + g] = s[r];
                        a.zeros[(long long)row * a.G + g] = (uint8_t)z[r];
                    }
                }
            }
            const float ut = invd[t];
            const float *urow = Us + t * B + 32 * q + lane;
#pragma unroll
            for (int r = 0; r < ROWS; ++r) {
                const float wt = __shfl_sync(0xffffffffu, w[r][0], o);
                const float v = fmaf(wt, is[r], z[r]);
                const float c = fminf(fmaxf(rintf(v), 0.f), fmaxq);
                const float wq = s[r] * (c - z[r]);
                const float e = (wt - wq) * ut;
                if (lane == o) {
                    cvc[r] = c;
                    evc[r] = e;
                }
                if (lane > o) w[r][0] = fmaf(-e, urow[0], w[r][0]);
#pragma unroll
                for (int sl = 1; sl < NSLOT; ++sl)
                    if (q + sl < NSLOT) w[r][sl] = fmaf(-e, urow[32 * sl], w[r][sl]);
            }
        }
        // slot q is final: its errors (for the lazy update), codes and loss share
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int row = row0 + r;
            if (rv[r]) {
                const float eh = tcg::to_tf32(evc[r]);
                a.err[(long long)row * a.lde + 32 * q + lane] = eh;
                a.err_lo[(long long)row * a.lde + 32 * q + lane] = tcg::to_tf32(evc[r] - eh);
            }
            cb[r * B + 32 * q + lane] = (uint8_t)(int)cvc[r];
            lacc[r] += (double)evc[r] * (double)evc[r];
#pragma unroll
            for (int sl = 0; sl + 1 < NSLOT; ++sl) w[r][sl] = w[r][sl + 1];
            w[r][NSLOT - 1] = 0.f;
        }
    }
    if (a.loss) {
#pragma unroll
        for (int r = 0; r < ROWS; ++r) {
            const int row = row0 + r;
            const double l = warp_sum_d(lacc[r]);
            if (lane == 0 && rv[r]) {
                if (j0 == 0) a.loss[row] = l;
                else a.loss[row] += l;
            }
        }
    }
    __syncwarp();
    const int bits = a.bits;
    const int wpp = B * bits / 32;  // words per row for this panel
#pragma unroll
    for (int r = 0; r < ROWS; ++r) {
        const int row = row0 + r;
        if (!rv[r] || lane >= wpp) continue;
        const int bit0 = lane * 32;
        const int cfirst = bit0 / bits, clast = min(B - 1, (bit0 + 31) / bits);
        uint32_t word = 0;
        for (int c = cfirst; c <= clast; ++c) {
            const int pos = c * bits - bit0;
            const uint32_t code = cb[r * B + c];
            word |= pos >= 0 ? (code << pos) : (code >> (-pos));
        }
        a.codes[(long long)row * a.ldcodes + (long long)j0 * bits / 32 + lane] = word;
    }
}

constexpr int COLLOOP_ROWS = 2;
constexpr int COLLOOP_THREADS = 256;

template <int NSLOT>
inline size_t colloop_smem() {
    constexpr int B = 32 * NSLOT;
    return (size_t)B * B * 4 + B * 4 + (COLLOOP_THREADS / 32) * COLLOOP_ROWS * B;
}

template <int NSLOT>
inline int colloop_launch(const ColloopArgs &a, cudaStream_t s) {
    const size_t smem = colloop_smem<NSLOT>();
    GPTQ_SMEM_LIMIT((colloop_kernel<NSLOT, COLLOOP_ROWS>), smem);
    const int rows_per_cta = (COLLOOP_THREADS / 32) * COLLOOP_ROWS;
    colloop_kernel<NSLOT, COLLOOP_ROWS>
        <<<ceil_div(a.m, rows_per_cta), COLLOOP_THREADS, smem, s>>>(a);
    return launch_status();
}

// R[t, i] = Wc[i, n + t]: the extra columns, transposed to r x m.
__global__ void extract_R_kernel(const float *Wc, long long ldw, int m, int n, int r, float *R) {
    const long long total = (long long)r * m;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int t = (int)(idx / m), i = (int)(idx % m);
        R[idx] = Wc[(long long)i * ldw + n + t];
    }
}

// The sweep over all panels of a prepared working copy Wc (m x N, first n columns quantized).
// Width of the outer blocks of the two-level lazy update: 1024 columns (or n if smaller) when
// every group that starts inside an outer block also ends inside it, i.e. for one group per
// row or a group length dividing 1024 (group statistics then see fully updated weights);
// otherwise one level only (outer width = B). Always <= QUANT_OUTER_MAX, the row stride the
// workspace reserves for the errors.
constexpr int QUANT_OUTER_MAX = 1024;
inline int outer_block(int n, int gs, int B) {
    const int ob = (gs >= n || QUANT_OUTER_MAX % gs == 0) ? QUANT_OUTER_MAX : B;
    return ob < n ? ob : n;
}

// The sweep over all panels of a prepared working copy Wc (m x N, first n columns quantized).
// Lazy updates are two-level (GPTQ's lazy block update, applied at two widths; GPTQ-2D,
// Theorem 1: any order that respects the feedback dependencies rounds the same):
//   after each panel of B columns:      Wc[:, panel_end:outer_end] -= Err_panel U[panel, ...]
//   after each outer block of OB cols:  Wc[:, outer_end:N]         -= Err_outer U[outer, ...]
// so the columns far to the right receive one K = OB product per outer block instead of OB/B
// products with K = B. Err holds m x OB floats.
inline int sweep_layer(float *Wc, long long ldw, int m, int n, int N, const float *U,
                       long long ldu, int bits, int group_size, int B, uint32_t *codes,
                       float *scales, uint8_t *zeros, double *loss, float *Err, float *Err_lo,
                       cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_SWEEP);
    const int gs = group_size ? group_size : n;
    const int OB = outer_block(n, gs, B);
    ColloopArgs a;
    a.Wc = Wc; a.ldw = ldw; a.U = U; a.ldu = ldu; a.m = m; a.n = n;
    a.bits = bits; a.gs = gs;
    a.codes = codes; a.ldcodes = (long long)n * bits / 32;
    a.scales = scales; a.zeros = zeros; a.G = group_size ? n / group_size : 1;
    a.lde = OB; a.loss = loss;
    for (int o0 = 0; o0 < n; o0 += OB) {
        const int o1 = o0 + OB < n ? o0 + OB : n;
        for (int j0 = o0; j0 < o1; j0 += B) {
            a.j0 = j0;
            a.err = Err + (j0 - o0);
            a.err_lo = Err_lo + (j0 - o0);
            int st;
            switch (B) {
                case 32: st = colloop_launch<1>(a, s); break;
                case 64: st = colloop_launch<2>(a, s); break;
                default: st = colloop_launch<4>(a, s); break;
            }
            if (st) return st;
            const int j1 = j0 + B;
            if (j1 < o1) {
                // inner: Wc[:, j1:o1] -= Err_panel (m x B) * U[j0:j1, j1:o1]
                auto p = gemm_args<float, float>(m, o1 - j1, B, Err + (j0 - o0), OB, 0,
                                                 U + (long long)j0 * ldu + j1, ldu, 0, Wc + j1,
                                                 ldw, -1.f, 1.f);
                p.a_lo = Err_lo + (j0 - o0);
                if (int st2 = gemm_f32(p, s)) return st2;
            }
        }
        if (o1 < N) {
            // outer: Wc[:, o1:N] -= Err_outer (m x (o1 - o0)) * U[o0:o1, o1:N]
            auto p = gemm_args<float, float>(m, N - o1, o1 - o0, Err, OB, 0,
                                             U + (long long)o0 * ldu + o1, ldu, 0, Wc + o1, ldw,
                                             -1.f, 1.f);
            p.a_lo = Err_lo;
            if (int st2 = gemm_f32(p, s)) return st2;
        }
    }
    return GPTQ_OK;
}

}  // namespace gptq
