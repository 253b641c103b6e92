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
    float *Wc;          // m x N working weights (row stride ldw); a finished panel keeps
                        // its codes there as bytes (first CPL bytes of each CPL-column slot)
    long long ldw;
    const float *U;     // n x N upper factor rows (row stride ldu)
    long long ldu;
    int m, n;           // rows, quantized columns
    int j0;             // first column of this panel
    int bits;
    int gs;             // group length (n when there is one group per row)
    float *scales;      // m x G
    uint8_t *zeros;     // m x G
    int G;
    float *err;         // errors of this panel: m x B block at err (row stride lde), as the
    float *err_lo;      // tf32 pair hi = tf32(e) (err), lo = tf32(e - hi) (err_lo) that the
    long long lde;      // lazy update's tensor-core product takes without converting them
    double *loss;       // m or nullptr
    int pdl;            // launched as a programmatic dependent (its U block loads before the
                        // previous kernel of the stream has finished; U is not written there)
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

constexpr int COLLOOP_THREADS = 64;

// One warp = 32 / LPR rows; the LPR = B / CPL lanes of a row each hold CPL (16) consecutive
// columns of the panel in registers (lane k of the row: columns CPL k .. CPL k + CPL-1, "slot"
// k), so that the rounding of a column is evaluated by LPR lanes per row and every lane applies
// at most CPL updates per column. The panel's U block sits in shared memory (rows from their
// diagonal slot on, zeros to the left of it; 4 floats of padding after every slot, so that the
// lanes of a row, which read 16 bytes each from their own slot, hit different banks). Per
// column t = CPL q + o: the owner lane (k = q) broadcasts register o to its row's lanes by
// shuffle, every lane of the row evaluates the rounding, and each lane applies -e * U[t, col]
// to its own columns after t, the next column first (its new value is the next step's
// shuffle). Lanes without work in a step multiply by a zero error instead of branching (U is
// finite, the zeros left of the diagonal included), so the warp never diverges. The owner keeps
// e in the column's register, so that at the end of the panel every register holds the error
// of its column; the codes go to the panel's own columns of Wc as bytes (those columns are
// final) and are bit-packed once after the sweep. SMALLG: groups shorter than a slot, whose
// boundaries fall inside it.
constexpr int COLLOOP_CPL = 16;  // columns per lane
template <int B>
struct ColloopShape {
    static constexpr int CPL = COLLOOP_CPL;
    static constexpr int LPR = B / CPL;        // lanes per row
    static constexpr int RPW = 32 / LPR;       // rows per warp
    static constexpr int LDU = B + 4 * LPR;    // padded row of the U block, in floats
    static __host__ __device__ constexpr int col(int c) { return c + 4 * (c / CPL); }
};

template <int B, bool SMALLG>
__global__ __launch_bounds__(COLLOOP_THREADS, 1) void colloop_kernel(ColloopArgs a) {
    using S = ColloopShape<B>;
    constexpr int CPL = S::CPL, LPR = S::LPR, RPW = S::RPW, LDU = S::LDU;
    extern __shared__ float sm[];
    float *Us = sm;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nwarps = blockDim.x >> 5;
    const int k = lane % LPR;
    const int row = (blockIdx.x * nwarps + warp) * RPW + lane / LPR;
    const bool rv = row < a.m;
    const int j0 = a.j0;
    pdl_launch_next();
    // U block: slot q's rows (CPL q .. CPL q + CPL-1) hold zeros left of column CPL q; from there on
    // cp.async when the rows are 16-byte aligned, else plain loads
    for (int q = 1; q < LPR; ++q) {
        const int f4 = CPL * q / 4;  // float4s of a row left of its diagonal slot
        for (int c = tid; c < CPL * f4; c += blockDim.x) {
            const int rr = CPL * q + c / f4, cc = (c % f4) * 4;
            *reinterpret_cast<float4 *>(Us + rr * LDU + S::col(cc)) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    const bool async_u = ((reinterpret_cast<uintptr_t>(a.U) | (uintptr_t)(a.ldu * 4)) & 15u) == 0;
    if (async_u) {
#pragma unroll
        for (int q = 0; q < LPR; ++q) {
            const int w4 = (B - CPL * q) / 4;  // float4s per row from the diagonal slot on
            for (int c = tid; c < CPL * w4; c += blockDim.x) {
                const int rr = CPL * q + c / w4, cc = CPL * q + (c % w4) * 4;
                const unsigned d =
                    static_cast<unsigned>(__cvta_generic_to_shared(Us + rr * LDU + S::col(cc)));
                const float *src = a.U + (long long)(j0 + rr) * a.ldu + j0 + cc;
                asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
            }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    } else {
        for (int idx = tid; idx < B * B; idx += blockDim.x) {
            const int rr = idx / B, cc = idx % B;
            if (cc >= (rr & ~(CPL - 1)))
                Us[rr * LDU + S::col(cc)] = a.U[(long long)(j0 + rr) * a.ldu + j0 + cc];
        }
    }
    // the next panel's U block into L2 while this panel runs (one CTA asks for it)
    if (blockIdx.x == 0 && j0 + 2 * B <= a.n) {
        for (int rr = tid; rr < B; rr += blockDim.x) {
            const float *p = a.U + (long long)(j0 + B + rr) * a.ldu + j0 + B;
#pragma unroll
            for (int c = 0; c < B; c += 32) asm volatile("prefetch.global.L2 [%0];" ::"l"(p + c));
        }
    }

    pdl_wait_prev();  // the weights (and grids) are the previous kernel's output

    float w[CPL];
    {
        const float *src = a.Wc + (long long)row * a.ldw + j0 + CPL * k;
        const bool vec = ((reinterpret_cast<uintptr_t>(a.Wc) | (uintptr_t)(a.ldw * 4)) & 15u) == 0;
        if (rv && vec) {
#pragma unroll
            for (int j = 0; j < CPL / 4; ++j) {
                const float4 v = reinterpret_cast<const float4 *>(src)[j];
                w[4 * j] = v.x; w[4 * j + 1] = v.y; w[4 * j + 2] = v.z; w[4 * j + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int r = 0; r < CPL; ++r) w[r] = rv ? src[r] : 0.f;
        }
    }

    const int maxq = (1 << a.bits) - 1;
    const float fmaxq = (float)maxq;
    const int gs = a.gs;
    const bool groups_in_panel = gs <= B;  // then B % gs == 0
    const int gmask = groups_in_panel ? gs - 1 : 0;
    float s = 1.f, is = 1.f, z = 0.f;
    if (!groups_in_panel) {
        // one group spans several panels; its grid was computed at its first panel
        const int g = j0 / gs;
        if (rv) {
            s = a.scales[(long long)row * a.G + g];
            z = (float)a.zeros[(long long)row * a.G + g];
            is = __frcp_rn(s);
        }
    }

    // grid of the group that starts at panel column t, from the current weights of its columns
    auto group_grid = [&](int t) {
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int r = 0; r < CPL; ++r) {
            if ((unsigned)(CPL * k + r - t) < (unsigned)gs) {
                mn = fminf(mn, w[r]);
                mx = fmaxf(mx, w[r]);
            }
        }
#pragma unroll
        for (int x = 1; x < LPR; x <<= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, x));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, x));
        }
        grid_from_range(mn, mx, fmaxq, s, is, z);
        if (k == 0 && rv) {
            const int g = (j0 + t) / gs;
            a.scales[(long long)row * a.G + g] = s;
            a.zeros[(long long)row * a.G + g] = (uint8_t)z;
        }
    };

    // 1 / U[t, t] for every row of the block, once it has arrived
    if (async_u) asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    __syncthreads();
    float *invd = Us + B * LDU;
    for (int t = tid; t < B; t += blockDim.x) invd[t] = __frcp_rn(Us[t * LDU + S::col(t)]);
    __syncthreads();

    // Rounding with the magic constant 1.5 * 2^23: fmaf(w, 1/s, z + MAGIC) - (z + MAGIC) is the
    // product w/s + z rounded once, to the nearest integer with ties to even (|w/s + z| < 2^22;
    // anything larger clamps the same way), minus z; clamped to [-z, maxq - z] it is c - z.
    constexpr float MAGIC = 12582912.f;
    // With DEFER the updates of column t's error to the lane's other columns are applied in the
    // next step, behind that step's chain (its rounding, the next column's update and shuffle):
    // only the column the next shuffle reads needs them first. Groups shorter than a slot
    // (SMALLG) read the registers between steps and take every update at once instead.
    constexpr bool DEFER = !SMALLG;
    uint32_t cw[CPL / 4] = {};  // codes of this lane's columns, one byte each
    const int src_base = lane & ~(LPR - 1);
    float wt = __shfl_sync(0xffffffffu, w[0], src_base);
#pragma unroll 1
    for (int q = 0; q < LPR; ++q) {
        const int src = src_base | q;
        const bool own = k == q, after = k >= q, upto = k > q;
        const bool last = q + 1 == LPR;
        const float *urow = Us + CPL * q * LDU + S::col(CPL * k);  // row CPL q, this lane's slot
        if (groups_in_panel && ((CPL * q) & gmask) == 0) group_grid(CPL * q);
        const float zm = z + MAGIC, nz = -z, hz = fmaxq - z;
        float uts[CPL];  // 1 / U[t, t] for the slot's columns
#pragma unroll
        for (int j = 0; j < CPL / 4; ++j) {
            const float4 x = reinterpret_cast<const float4 *>(invd + CPL * q)[j];
            uts[4 * j] = x.x; uts[4 * j + 1] = x.y; uts[4 * j + 2] = x.z; uts[4 * j + 3] = x.w;
        }
        float4 un[CPL / 4];
#pragma unroll
        for (int j = 0; j < CPL / 4; ++j) un[j] = reinterpret_cast<const float4 *>(urow)[j];
        float up[CPL];            // the previous step's row of U (DEFER)
        float eap = 0.f, eup = 0.f;  // and its masked errors
#pragma unroll
        for (int o = 0; o < CPL; ++o) {
            if (SMALLG && o > 0 && groups_in_panel && (o & gmask) == 0) group_grid(CPL * q + o);
            const float zmo = SMALLG ? z + MAGIC : zm, nzo = SMALLG ? -z : nz,
                        hzo = SMALLG ? fmaxq - z : hz;
            const float ut = uts[o];
            float u[CPL];
#pragma unroll
            for (int j = 0; j < CPL / 4; ++j) {
                u[4 * j] = un[j].x; u[4 * j + 1] = un[j].y; u[4 * j + 2] = un[j].z; u[4 * j + 3] = un[j].w;
            }
            if (o + 1 < CPL) {
                // the next row of U while this column is rounded
#pragma unroll
                for (int j = 0; j < CPL / 4; ++j)
                    un[j] = reinterpret_cast<const float4 *>(urow + (o + 1) * LDU)[j];
            }
            const int rn = (o + 1) & (CPL - 1);  // the column the next shuffle reads
            if (DEFER && o > 0) w[rn] = fmaf(-(rn > o - 1 ? eap : eup), up[rn], w[rn]);
            // its multiplier, scaled by 1 / U[t, t] and masked to the lanes that hold it still
            // unquantized (off the chain: it waits only for U)
            const float un_next = ((o + 1 < CPL) ? after : upto) ? u[rn] * ut : 0.f;
            const float d = fminf(fmaxf(fmaf(wt, is, zmo) - zmo, nzo), hzo);  // c - z
            const float e1 = fmaf(-s, d, wt);                                 // w_t - q_t
            // the next column first: its value is the next step's shuffle (it takes
            // e1 * (U[t, col] / U[t, t]), the other columns (e1 / U[t, t]) * U[t, col]: the same
            // product, rounded in another order)
            w[rn] = fmaf(-e1, un_next, w[rn]);
            if (o + 1 < CPL) wt = __shfl_sync(0xffffffffu, w[rn], src);
            else if (!last) wt = __shfl_sync(0xffffffffu, w[0], src + 1);
            if (DEFER && o > 0) {
#pragma unroll
                for (int r = 0; r < CPL; ++r) {
                    if (r == rn || r == o) continue;  // o: the previous step's next column
                    w[r] = fmaf(-(r > o - 1 ? eap : eup), up[r], w[r]);
                }
            }
            const float e = e1 * ut;
            const float ea = after ? e : 0.f;  // for this lane's columns after t
            const float eu = upto ? e : 0.f;   // for its columns up to t
            if (!DEFER) {
#pragma unroll
                for (int r = 0; r < CPL; ++r) {
                    if (r == rn) continue;
                    w[r] = fmaf(-(r > o ? ea : eu), u[r], w[r]);
                }
            }
            w[o] = own ? e : w[o];
            const uint32_t code = __float_as_uint(d + zmo) & 0xffu;  // MAGIC + c
            cw[o >> 2] |= (own ? code : 0u) << (8 * (o & 3));
            if (DEFER) {
                eap = ea;
                eup = eu;
#pragma unroll
                for (int r = 0; r < CPL; ++r) up[r] = u[r];
            }
        }
        if (DEFER) {
            // the slot's last column reaches the lane's other columns before the next slot
#pragma unroll
            for (int r = 1; r < CPL; ++r) w[r] = fmaf(-eup, up[r], w[r]);
        }
    }

    // the registers now hold the panel's errors: tf32 pairs for the lazy update, their squares
    // for the loss; the codes go to the first CPL bytes of this lane's CPL columns of Wc
    float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int r = 0; r < CPL; ++r) l4[r & 3] = fmaf(w[r], w[r], l4[r & 3]);
    double l = ((double)l4[0] + (double)l4[1]) + ((double)l4[2] + (double)l4[3]);
#pragma unroll
    for (int x = 1; x < LPR; x <<= 1) l += __shfl_xor_sync(0xffffffffu, l, x);
    if (!rv) return;
    float *eh = a.err + (long long)row * a.lde + CPL * k;
    float *el = a.err_lo + (long long)row * a.lde + CPL * k;
    uint32_t *cdst = reinterpret_cast<uint32_t *>(a.Wc + (long long)row * a.ldw + j0 + CPL * k);
    const bool vec = ((reinterpret_cast<uintptr_t>(a.err) | reinterpret_cast<uintptr_t>(a.err_lo) |
                       (uintptr_t)(a.lde * 4) | reinterpret_cast<uintptr_t>(a.Wc) |
                       (uintptr_t)(a.ldw * 4)) & 15u) == 0;
    if (vec) {
#pragma unroll
        for (int j = 0; j < CPL / 4; ++j) {
            float4 h, lo;
            h.x = tcg::to_tf32(w[4 * j]);     lo.x = tcg::to_tf32(w[4 * j] - h.x);
            h.y = tcg::to_tf32(w[4 * j + 1]); lo.y = tcg::to_tf32(w[4 * j + 1] - h.y);
            h.z = tcg::to_tf32(w[4 * j + 2]); lo.z = tcg::to_tf32(w[4 * j + 2] - h.z);
            h.w = tcg::to_tf32(w[4 * j + 3]); lo.w = tcg::to_tf32(w[4 * j + 3] - h.w);
            reinterpret_cast<float4 *>(eh)[j] = h;
            reinterpret_cast<float4 *>(el)[j] = lo;
        }
        if constexpr (CPL == 16) *reinterpret_cast<uint4 *>(cdst) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        else if constexpr (CPL == 8) *reinterpret_cast<uint2 *>(cdst) = make_uint2(cw[0], cw[1]);
        else for (int j = 0; j < CPL / 4; ++j) cdst[j] = cw[j];
    } else {
#pragma unroll
        for (int r = 0; r < CPL; ++r) {
            const float h = tcg::to_tf32(w[r]);
            eh[r] = h;
            el[r] = tcg::to_tf32(w[r] - h);
        }
#pragma unroll
        for (int j = 0; j < CPL / 4; ++j) cdst[j] = cw[j];
    }
    if (a.loss && k == 0) {
        if (j0 == 0) a.loss[row] = l;
        else a.loss[row] += l;
    }
}

// Bit-packs the codes that the column loop left as bytes at the start of every cpl-column slot
// of Wc (the codes of columns cpl*i .. cpl*i + cpl-1 in the first cpl bytes of Wc[row, cpl*i];
// cpl = 4, 8, 16 or 32). One thread per row and 32 columns: their 32 codes fill exactly `bits`
// words of the packed row (code c at bits [c * bits, (c + 1) * bits) of the row's stream,
// little-endian words).
__global__ void pack_sweep_codes_kernel(const float *Wc, long long ldw, long long m, int n,
                                        int bits, int cpl, uint32_t *codes, long long ldcodes) {
    const int chunks = n / 32;
    const long long total = m * chunks;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const long long row = idx / chunks;
        const int ch = (int)(idx % chunks);
        const uint32_t *src = reinterpret_cast<const uint32_t *>(Wc + row * ldw + 32 * ch);
        uint32_t cw[8];  // codes 4j .. 4j+3: word (4j mod cpl) / 4 of the slot at 4j - 4j mod cpl
#pragma unroll
        for (int j = 0; j < 8; ++j) cw[j] = src[((4 * j) & ~(cpl - 1)) + (((4 * j) & (cpl - 1)) >> 2)];
        uint32_t *dst = codes + row * ldcodes + (long long)ch * bits;
        unsigned long long buf = 0;
        int nb = 0, wi = 0;
#pragma unroll
        for (int o = 0; o < 32; ++o) {
            buf |= (unsigned long long)((cw[o >> 2] >> (8 * (o & 3))) & 0xffu) << nb;
            nb += bits;
            if (nb >= 32) {
                dst[wi++] = (uint32_t)buf;
                buf >>= 32;
                nb -= 32;
            }
        }
    }
}

// Grids of groups that span several panels (group length > B), computed at the group's first
// panel from the weights of the whole group as they stand then: one warp per row.
__global__ void group_grid_kernel(const float *Wc, long long ldw, int m, int c0, int c1, int bits,
                                  float *scales, uint8_t *zeros, int G, int g) {
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= m) return;
    const float *src = Wc + (long long)row * ldw;
    float mn = INFINITY, mx = -INFINITY;
    for (int c = c0 + lane; c < c1; c += 32) {
        const float x = src[c];
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
    }
    mn = warp_min(mn);
    mx = warp_max(mx);
    float s, is, z;
    grid_from_range(mn, mx, (float)((1 << bits) - 1), s, is, z);
    if (lane == 0) {
        scales[(long long)row * G + g] = s;
        zeros[(long long)row * G + g] = (uint8_t)z;
    }
}

template <int B>
inline size_t colloop_smem() {
    return ((size_t)B * ColloopShape<B>::LDU + B) * 4;  // U block + 1 / U[t, t]
}

template <int B>
inline int colloop_launch(const ColloopArgs &a, cudaStream_t s) {
    if (a.gs > B && a.j0 % a.gs == 0) {
        const int c1 = a.j0 + a.gs < a.n ? a.j0 + a.gs : a.n;
        group_grid_kernel<<<ceil_div(a.m, 8), 256, 0, s>>>(a.Wc, a.ldw, a.m, a.j0, c1, a.bits,
                                                           a.scales, a.zeros, a.G, a.j0 / a.gs);
        if (int st = launch_status()) return st;
    }
    const size_t smem = colloop_smem<B>();
    const int rows_per_cta = COLLOOP_THREADS / ColloopShape<B>::LPR;
    const dim3 grid(ceil_div(a.m, rows_per_cta));
    if (a.gs < ColloopShape<B>::CPL) {
        GPTQ_SMEM_LIMIT((colloop_kernel<B, true>), smem);
        return launch_kernel(colloop_kernel<B, true>, grid, dim3(COLLOOP_THREADS), smem, s,
                             a.pdl != 0, a);
    }
    GPTQ_SMEM_LIMIT((colloop_kernel<B, false>), smem);
    return launch_kernel(colloop_kernel<B, false>, grid, dim3(COLLOOP_THREADS), smem, s,
                         a.pdl != 0, a);
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

// Rows r0 .. r1-1 of U, columns c0 .. N-1, split into tf32 pairs (round to nearest, as the
// tensor-core product's converters would): Uh[i, c] = tf32(U[r0 + i, c]),
// Ul[i, c] = tf32(U[r0 + i, c] - Uh[i, c]) (row stride N).
__global__ void split_band_kernel(const float *U, long long ldu, int r0, int r1, int c0, int N,
                                  float *Uh, float *Ul) {
    const int w4 = (N - c0) / 4;  // c0 and N are multiples of 4
    const long long total = (long long)(r1 - r0) * w4;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int i = (int)(idx / w4), c = c0 + 4 * (int)(idx % w4);
        const float4 v = *reinterpret_cast<const float4 *>(U + (long long)(r0 + i) * ldu + c);
        float4 h, l;
        h.x = tcg::to_tf32(v.x); l.x = tcg::to_tf32(v.x - h.x);
        h.y = tcg::to_tf32(v.y); l.y = tcg::to_tf32(v.y - h.y);
        h.z = tcg::to_tf32(v.z); l.z = tcg::to_tf32(v.z - h.z);
        h.w = tcg::to_tf32(v.w); l.w = tcg::to_tf32(v.w - h.w);
        *reinterpret_cast<float4 *>(Uh + (long long)i * N + c) = h;
        *reinterpret_cast<float4 *>(Ul + (long long)i * N + c) = l;
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
                       float *Uh, float *Ul, cudaStream_t s) {
    KtStageScope stage(GPTQ_KT_SWEEP);
    const int gs = group_size ? group_size : n;
    const int OB = outer_block(n, gs, B);
    ColloopArgs a;
    a.Wc = Wc; a.ldw = ldw; a.U = U; a.ldu = ldu; a.m = m; a.n = n;
    a.bits = bits; a.gs = gs;
    a.scales = scales; a.zeros = zeros; a.G = group_size ? n / group_size : 1;
    a.lde = OB; a.loss = loss;
    // the band of U that an outer block's updates read, split once (when U's rows allow
    // 16-byte vectors and the caller gave room for it)
    const bool band = Uh && Ul && ldu % 4 == 0 && N % 4 == 0 &&
                      ((reinterpret_cast<uintptr_t>(U) | reinterpret_cast<uintptr_t>(Uh) |
                        reinterpret_cast<uintptr_t>(Ul)) & 15u) == 0;
    for (int o0 = 0; o0 < n; o0 += OB) {
        const int o1 = o0 + OB < n ? o0 + OB : n;
        if (band) {
            split_band_kernel<<<4 * device_sm_count(), 256, 0, s>>>(U, ldu, o0, o1, o0, N, Uh, Ul);
            if (int st = launch_status()) return st;
        }
        // B operand of an update reading U[j, c] (j in this outer block): the band's pair
        auto bh = [&](int j, int c) { return Uh + (long long)(j - o0) * N + c; };
        auto bl = [&](int j, int c) { return Ul + (long long)(j - o0) * N + c; };
        for (int j0 = o0; j0 < o1; j0 += B) {
            a.j0 = j0;
            a.pdl = j0 > 0;  // the first panel's predecessor may still be writing U
            a.err = Err + (j0 - o0);
            a.err_lo = Err_lo + (j0 - o0);
            int st;
            switch (B) {
                case 32: st = colloop_launch<32>(a, s); break;
                case 64: st = colloop_launch<64>(a, s); break;
                default: st = colloop_launch<128>(a, s); break;
            }
            if (st) return st;
            const int j1 = j0 + B;
            if (j1 < o1) {
                // inner: Wc[:, j1:o1] -= Err_panel (m x B) * U[j0:j1, j1:o1]
                auto p = band ? gemm_args<float, float>(m, o1 - j1, B, Err + (j0 - o0), OB, 0,
                                                        bh(j0, j1), N, 0, Wc + j1, ldw, -1.f, 1.f)
                              : gemm_args<float, float>(m, o1 - j1, B, Err + (j0 - o0), OB, 0,
                                                        U + (long long)j0 * ldu + j1, ldu, 0,
                                                        Wc + j1, ldw, -1.f, 1.f);
                p.a_lo = Err_lo + (j0 - o0);
                if (band) {
                    p.b_lo = bl(j0, j1);
                    p.b_full = U + (long long)j0 * ldu + j1;
                    p.ldb_full = ldu;
                }
                p.pdl = 1;
                if (int st2 = gemm_f32(p, s)) return st2;
            }
        }
        if (o1 < N) {
            // outer: Wc[:, o1:N] -= Err_outer (m x (o1 - o0)) * U[o0:o1, o1:N]
            auto p = band ? gemm_args<float, float>(m, N - o1, o1 - o0, Err, OB, 0, bh(o0, o1), N,
                                                    0, Wc + o1, ldw, -1.f, 1.f)
                          : gemm_args<float, float>(m, N - o1, o1 - o0, Err, OB, 0,
                                                    U + (long long)o0 * ldu + o1, ldu, 0, Wc + o1,
                                                    ldw, -1.f, 1.f);
            p.a_lo = Err_lo;
            if (band) {
                p.b_lo = bl(o0, o1);
                p.b_full = U + (long long)o0 * ldu + o1;
                p.ldb_full = ldu;
            }
            p.pdl = 1;
            if (int st2 = gemm_f32(p, s)) return st2;
        }
    }
    pack_sweep_codes_kernel<<<4 * device_sm_count(), 256, 0, s>>>(Wc, ldw, m, n, bits, COLLOOP_CPL,
                                                                  codes, (long long)n * bits / 32);
    return launch_status();
}

}  // namespace gptq
