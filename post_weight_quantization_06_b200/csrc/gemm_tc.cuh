// fp32-accurate GEMM on the tcgen05 tensor cores (kind::tf32, three MMAs per K step):
//   C = alpha * op(A) op(B) + beta * C          (M x N, fp32 in global memory)
//
// The factor and the lazy trailing update need fp32 accuracy: a plain tf32 product moves the
// pre-rounding values of the sweep by ~1e-3 grid steps. Each fp32 operand x is split into
// hi = x rounded to the nearest tf32 and lo = (x - hi) rounded to the nearest tf32
// (|lo| <= 2^-11 |x|); a b ~ a_hi b_hi + a_hi b_lo + a_lo b_hi, error ~2^-22 |a b|.
//
// Operand staging: TMA loads 32-deep K slices of both operands with the 128-byte swizzle;
// "K-major" when K is the contiguous index (one 128-row box), "MN-major" when M / N is (four
// 32-wide boxes). Converter warps then write lo next to the slice and overwrite the slice
// with hi (the split is elementwise, so it runs on the swizzled bytes as they are).
//
// Warp roles (320 threads, one CTA per SM, persistent over 128 x 128 output tiles):
//   warp 0     TMA producer, 3-stage ring of {A, A_lo, B, B_lo} (64 KB per stage)
//   warp 1     TMEM allocation and the MMA issuer (one thread); 3 x 4 MMAs per stage
//   warps 2-5  hi/lo converters
//   warps 6-9  epilogue: one row of the tile per thread (TMEM lane = row); per 32-column
//              slice either a bulk tensor store / add-reduction of alpha * acc through the C
//              map (beta 0 or 1) or a read-modify-write of C through shared memory
// Triangular operands: a_upper / a_lower / b_upper / b_lower restrict each tile's K range to
// where the operand can be nonzero; the storage of the zero triangle must hold zeros.
// All mbarrier waits are bounded as in the Hessian kernel.
#pragma once

#include <cuda.h>

#include <cstdlib>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "hessian_tc.cuh"

namespace gptq {
namespace tcg {

using tc::desc_mn_sw128;
using tc::mbar_arrive;
using tc::mbar_expect_tx;
using tc::mbar_init;
using tc::mbar_wait;
using tc::mma_commit;
using tc::smem_u32;
using tc::tc_fence_after;
using tc::tc_fence_before;
using tc::tma_load_2d;
using tc::tmem_alloc;
using tc::tmem_dealloc;
using tc::tmem_relinquish;

constexpr int TILE = 128;
constexpr int BK = 32;                    // fp32 elements per K slice (128 bytes)
constexpr int STAGES = 3;
constexpr int SLICE_BYTES = TILE * BK * 4;          // 16 KB
constexpr int STAGE_BYTES = 4 * SLICE_BYTES;        // A, A_lo, B, B_lo
constexpr int CONV_WARPS = 4, EPI_WARPS = 4;
constexpr int CONV_PER = SLICE_BYTES / 16 / (CONV_WARPS * 32);   // float4 per converter thread
static_assert(CONV_PER * CONV_WARPS * 32 * 16 == SLICE_BYTES, "converter threads tile a slice");
constexpr int THREADS = 32 * (2 + CONV_WARPS + EPI_WARPS);
constexpr int TMEM_COLS = 2 * TILE;
// Per epilogue warp: a padded 32 x 33 staging slice (read-modify-write epilogue) or one 32 x 32
// slice in the 128-byte swizzle for the C tensor map; 1024-byte aligned for the swizzle.
constexpr size_t EPI_WARP_BYTES = 5120;
constexpr size_t EPI_OFFSET = (size_t)STAGES * STAGE_BYTES + 1024;   // after the barriers
constexpr size_t SMEM_BYTES = 1024 + EPI_OFFSET + (size_t)EPI_WARPS * EPI_WARP_BYTES;
static_assert(EPI_WARP_BYTES % 1024 == 0 && EPI_WARP_BYTES >= 32 * 33 * 4, "epilogue buffer");
static_assert(SMEM_BYTES <= 232448, "fits the opt-in shared memory of one CTA");

__host__ __device__ constexpr uint32_t idesc_tf32(int a_mn, int b_mn) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(TILE >> 3) << 17) | ((uint32_t)(TILE >> 4) << 24);
}

// K-major operand, 128-byte swizzle: rows of 32 fp32 (128 B), 8-row groups 1024 B apart.
__device__ __forceinline__ uint64_t desc_k_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;                         // LBO (unused for swizzled K-major)
    d |= (uint64_t)((1024 >> 4) & 0x3FFFu) << 32;   // SBO: next 8 rows
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// MN-major operand of tf32: the only MN-major layout the tensor cores take for 32-bit
// elements is the 128-byte swizzle with 32-byte atoms (layout type 1), whose pattern repeats
// every 4 K rows. Rows are 128 B (32 M/N elements); 4-row groups are 512 B apart; the 32-wide
// M/N chunks (one TMA box of BK rows each) are BK * 128 B apart.
__device__ __forceinline__ uint64_t desc_mn32_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(((BK * 128) >> 4) & 0x3FFFu) << 16;  // LBO: next 32 M/N elements
    d |= (uint64_t)((512 >> 4) & 0x3FFFu) << 32;         // SBO: next 4 K rows
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)1 << 61;                               // 128B swizzle, 32B atoms
    return d;
}

// Round to the nearest tf32 value (kept as an fp32 bit pattern with the low 13 bits zero).
__device__ __forceinline__ float to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

__device__ __forceinline__ void mma_tf32(uint32_t dtmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float *v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct TcGemmParams {
    int M, N, K;
    float *C;
    long long ldc;
    float alpha, beta;
    int a_mn, b_mn;     // 1: operand is MN-major (M / N contiguous), 0: K-major
    int c_upper, a_upper, a_lower, b_upper, b_lower;
    int tiles_m, tiles_n;
    long long wait_limit;
    int c_tma;          // 1: beta is 0 or 1 and cmap covers C; slices may leave by tensor store /
                        // tensor add-reduction instead of a read-modify-write
    const int *skip;    // when set and *skip != 0 the launch does nothing
    int a_split;        // 1: A comes split (amap: tf32 hi, alomap: lo); only B is converted
    int b_split;        // 1: B comes split (bmap: tf32 hi, blomap: lo); with a_split as well
                        // nothing is converted and the MMA takes the slices as they land
};

// Bulk tensor writes of one 32 x 32 slice from shared memory (128-byte swizzle) through the C
// map: a plain store (beta = 0) or an fp32 add-reduction performed in L2 (beta = 1; one
// rounding of C + value, as the read-modify-write does).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}
__device__ __forceinline__ void tma_add_2d(const CUtensorMap *map, const void *src, int x, int y) {
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the bulk operations of this thread have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// K range [kb, ke) (multiples of BK) of output tile (ti, tj).
__device__ __forceinline__ void tile_k_range(const TcGemmParams &p, int ti, int tj, int &kb,
                                             int &ke) {
    int b = 0, e = p.K;
    const int i0 = ti * TILE, j0 = tj * TILE;
    if (p.a_upper) b = max(b, i0);
    if (p.b_lower) b = max(b, j0);
    if (p.a_lower) e = min(e, i0 + TILE);
    if (p.b_upper) e = min(e, j0 + TILE);
    kb = (b / BK) * BK;
    ke = e;
}

// Number of output tiles: with c_upper only the tiles on or above the diagonal exist.
__host__ __device__ __forceinline__ int num_tiles(const TcGemmParams &p) {
    return p.c_upper ? p.tiles_n * (p.tiles_n + 1) / 2 : p.tiles_m * p.tiles_n;
}

// Output tile of linear index t, enumerated so that the tiles with the longest K range come
// first (the persistent CTAs take tiles round-robin, so equal-work tiles land in the same
// round): with b_upper the K range of column tile j grows with j, with a_upper it shrinks
// with the row tile i, and so on; c_upper enumerates the upper triangle row by row.
__device__ __forceinline__ void tile_of(const TcGemmParams &p, int t, int &ti, int &tj) {
    if (p.c_upper) { tc::tile_coords(t, p.tiles_n, ti, tj); return; }
    if (p.b_upper) { tj = p.tiles_n - 1 - t / p.tiles_m; ti = t % p.tiles_m; return; }
    if (p.b_lower) { tj = t / p.tiles_m; ti = t % p.tiles_m; return; }
    if (p.a_lower) { ti = p.tiles_m - 1 - t / p.tiles_n; tj = t % p.tiles_n; return; }
    ti = t / p.tiles_n;
    tj = t % p.tiles_n;
}

// The 32 values C(row_base + r, col), r < 32, of one epilogue warp's slice (0 where C is not
// written); all 32 reads are issued together (the compiler cannot move them across the
// slice's stores), so a read-modify-write costs one round trip per slice.
__device__ __forceinline__ void epi_load_c(const TcGemmParams &p, int row_base, int col,
                                           float (&cin)[32]) {
#pragma unroll
    for (int r = 0; r < 32; ++r) {
        const int row = row_base + r;
        const bool ok = row < p.M && col < p.N && !(p.c_upper && col < row);
        cin[r] = ok ? p.C[(long long)row * p.ldc + col] : 0.f;
    }
}

__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
               const __grid_constant__ CUtensorMap cmap, const __grid_constant__ CUtensorMap alomap,
               const __grid_constant__ CUtensorMap blomap, TcGemmParams p) {
    pdl_launch_next();  // the stream's next kernel may set itself up meanwhile
    if (p.skip) {       // before any barrier, TMEM or copy: every thread leaves
        pdl_wait_prev();
        if (*p.skip) return;
    }
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                       // TMA -> converters
    uint64_t *conv = bars + STAGES;              // converters -> MMA
    uint64_t *empty = bars + 2 * STAGES;         // MMA -> TMA
    uint64_t *acc_full = bars + 3 * STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    unsigned char *epi_base = base + EPI_OFFSET;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = num_tiles(p);
    const bool no_conv = p.a_split && p.b_split;  // both operands arrive split
    if (threadIdx.x == 0) {
        // the descriptors' first fetch overlaps the setup instead of the first TMA load
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&amap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&bmap)) : "memory");
        if (p.c_tma) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&cmap)) : "memory");
        if (p.a_split) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&alomap)) : "memory");
        if (p.b_split) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&blomap)) : "memory");
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&conv[s], CONV_WARPS);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], EPI_WARPS); }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait_prev();  // the operands and C are the previous kernel's output from here on

    if (warp == 0) {
        if (lane == 0) {
            long long it = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
                int ti, tj;
                tile_of(p, t, ti, tj);
                int kb, ke;
                tile_k_range(p, ti, tj, kb, ke);
                for (int k0 = kb; k0 < ke; k0 += BK, ++it) {
                    const int slot = (int)(it % STAGES);
                    if (*abort_flag) break;
                    if (!mbar_wait(&empty[slot], (uint32_t)((it / STAGES) & 1) ^ 1u, p.wait_limit)) {
                        report(GPTQ_ERR_TIMEOUT, 11);
                        *abort_flag = 1;
                        break;
                    }
                    unsigned char *st = base + slot * STAGE_BYTES;
                    mbar_expect_tx(&full[slot], (2 + p.a_split + p.b_split) * SLICE_BYTES);
                    if (p.a_mn) {
                        for (int q = 0; q < 4; ++q)
                            tma_load_2d(&amap, &full[slot], st + q * (BK * 128), ti * TILE + 32 * q, k0);
                        if (p.a_split)
                            for (int q = 0; q < 4; ++q)
                                tma_load_2d(&alomap, &full[slot], st + SLICE_BYTES + q * (BK * 128),
                                            ti * TILE + 32 * q, k0);
                    } else {
                        tma_load_2d(&amap, &full[slot], st, k0, ti * TILE);
                        if (p.a_split) tma_load_2d(&alomap, &full[slot], st + SLICE_BYTES, k0, ti * TILE);
                    }
                    unsigned char *sb = st + 2 * SLICE_BYTES;
                    if (p.b_mn) {
                        for (int q = 0; q < 4; ++q)
                            tma_load_2d(&bmap, &full[slot], sb + q * (BK * 128), tj * TILE + 32 * q, k0);
                        if (p.b_split)
                            for (int q = 0; q < 4; ++q)
                                tma_load_2d(&blomap, &full[slot], sb + SLICE_BYTES + q * (BK * 128),
                                            tj * TILE + 32 * q, k0);
                    } else {
                        tma_load_2d(&bmap, &full[slot], sb, k0, tj * TILE);
                        if (p.b_split) tma_load_2d(&blomap, &full[slot], sb + SLICE_BYTES, k0, tj * TILE);
                    }
                }
            }
            if (*abort_flag)
                for (long long j = it - 1; j >= 0 && j >= it - STAGES; --j)
                    mbar_wait(&full[j % STAGES], (uint32_t)((j / STAGES) & 1), p.wait_limit);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_tf32(p.a_mn, p.b_mn);
            long long it = 0, ch = 0;
            for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
                int ti, tj;
                tile_of(p, t, ti, tj);
                int kb, ke;
                tile_k_range(p, ti, tj, kb, ke);
                if (ke <= kb) continue;   // nothing to accumulate: the epilogue writes beta C
                const int b = (int)(ch & 1);
                if (!mbar_wait(&acc_empty[b], (uint32_t)((ch >> 1) & 1) ^ 1u, p.wait_limit)) {
                    report(GPTQ_ERR_TIMEOUT, 12);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t dt = tmem + (uint32_t)(b * TILE);
                for (int k0 = kb; k0 < ke; k0 += BK, ++it) {
                    const int slot = (int)(it % STAGES);
                    if (!mbar_wait(no_conv ? &full[slot] : &conv[slot], (uint32_t)((it / STAGES) & 1),
                                   p.wait_limit)) {
                        report(GPTQ_ERR_TIMEOUT, 13);
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(base + slot * STAGE_BYTES);
                    const uint32_t sal = sa + SLICE_BYTES, sbb = sa + 2 * SLICE_BYTES,
                                   sbl = sa + 3 * SLICE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 8; ++kk) {
                        const uint32_t offa = p.a_mn ? kk * 1024u : kk * 32u;
                        const uint32_t offb = p.b_mn ? kk * 1024u : kk * 32u;
                        const uint64_t ah = p.a_mn ? desc_mn32_sw128(sa + offa) : desc_k_sw128(sa + offa);
                        const uint64_t al = p.a_mn ? desc_mn32_sw128(sal + offa) : desc_k_sw128(sal + offa);
                        const uint64_t bh = p.b_mn ? desc_mn32_sw128(sbb + offb) : desc_k_sw128(sbb + offb);
                        const uint64_t bl = p.b_mn ? desc_mn32_sw128(sbl + offb) : desc_k_sw128(sbl + offb);
                        const uint32_t acc0 = (k0 > kb || kk > 0) ? 1u : 0u;
                        mma_tf32(dt, ah, bh, idesc, acc0);
                        mma_tf32(dt, ah, bl, idesc, 1u);
                        mma_tf32(dt, al, bh, idesc, 1u);
                    }
                    mma_commit(&empty[slot]);
                }
                mma_commit(&acc_full[b]);
                ++ch;
            }
            mma_commit(mma_done);
            mbar_wait(mma_done, 0, p.wait_limit);
        }
    } else if (warp < 2 + CONV_WARPS) {
        // hi / lo split of each staged slice
        const int cw = warp - 2;
        long long it = 0;
        for (int t = blockIdx.x; !no_conv && t < ntiles && !*abort_flag; t += gridDim.x) {
            int ti, tj;
            tile_of(p, t, ti, tj);
            int kb, ke;
            tile_k_range(p, ti, tj, kb, ke);
            for (int k0 = kb; k0 < ke; k0 += BK, ++it) {
                const int slot = (int)(it % STAGES);
                if (!mbar_wait(&full[slot], (uint32_t)((it / STAGES) & 1), p.wait_limit)) {
                    if (lane == 0) report(GPTQ_ERR_TIMEOUT, 14);
                    *abort_flag = 1;
                    break;
                }
                unsigned char *st = base + slot * STAGE_BYTES;
                // every thread splits CONV_PER float4 of each operand (of B alone when A came
                // split); all of its shared-memory loads go out first so that their latencies
                // overlap
                const int op0 = p.a_split ? 1 : 0, op1 = p.b_split ? 1 : 2;
                float4 x[2][CONV_PER];
#pragma unroll
                for (int op = 0; op < 2; ++op) {
                    if (op < op0 || op >= op1) continue;
                    const float4 *hi = reinterpret_cast<const float4 *>(st + op * 2 * SLICE_BYTES);
#pragma unroll
                    for (int u = 0; u < CONV_PER; ++u) x[op][u] = hi[cw * 32 + lane + u * CONV_WARPS * 32];
                }
#pragma unroll
                for (int op = 0; op < 2; ++op) {
                    if (op < op0 || op >= op1) continue;
                    float4 *hi = reinterpret_cast<float4 *>(st + op * 2 * SLICE_BYTES);
                    float4 *lo = reinterpret_cast<float4 *>(st + op * 2 * SLICE_BYTES + SLICE_BYTES);
#pragma unroll
                    for (int u = 0; u < CONV_PER; ++u) {
                        const int i = cw * 32 + lane + u * CONV_WARPS * 32;
                        const float4 v = x[op][u];
                        float4 h, l;
                        h.x = to_tf32(v.x); h.y = to_tf32(v.y); h.z = to_tf32(v.z); h.w = to_tf32(v.w);
                        l.x = to_tf32(v.x - h.x); l.y = to_tf32(v.y - h.y);
                        l.z = to_tf32(v.z - h.z); l.w = to_tf32(v.w - h.w);
                        lo[i] = l;
                        hi[i] = h;
                    }
                }
                // generic-proxy writes must be visible to the tensor cores' async proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(&conv[slot]);
            }
        }
    } else {
        // epilogue: C = alpha * acc + beta * C
        const int q = warp & 3;
        const bool rd = p.beta != 0.f;
        unsigned char *ebuf = epi_base + (size_t)(warp - 2 - CONV_WARPS) * EPI_WARP_BYTES;
        float *stage = reinterpret_cast<float *>(ebuf);
        long long ch = 0;
        for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
            int ti, tj;
            tile_of(p, t, ti, tj);
            int kb, ke;
            tile_k_range(p, ti, tj, kb, ke);
            const bool has_acc = ke > kb;
            // Each warp owns rows [32 q, 32 q + 32) of the tile (TMEM lanes 32 q ...).
            const int row_base = ti * TILE + 32 * q;
            // With beta 0 or 1, an accumulator and no diagonal cut, the slices leave through
            // the C map and C is never read here; otherwise C is read and written in place.
            const bool via_map = p.c_tma && has_acc && !(p.c_upper && ti == tj);
            // The read-modify-write path reads C ahead of the accumulator: the warp's rows of
            // the tile are requested into L2 and the first slice's values into registers before
            // the wait, each later slice's values right after the previous slice's stores.
            float cin[32];
            if (rd && !via_map) {
                const int prow = row_base + lane;
                if (prow < p.M) {
#pragma unroll
                    for (int c = 0; c < TILE / 32; ++c) {
                        const int pcol = tj * TILE + 32 * c;
                        if (pcol < p.N)
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(p.C + (long long)prow * p.ldc + pcol));
                    }
                }
                epi_load_c(p, row_base, tj * TILE + lane, cin);
            }
            int b = 0;
            if (has_acc) {
                b = (int)(ch & 1);
                if (!mbar_wait(&acc_full[b], (uint32_t)((ch >> 1) & 1), p.wait_limit)) {
                    if (lane == 0) report(GPTQ_ERR_TIMEOUT, 15);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
            }
            if (via_map) {
#pragma unroll 1
                for (int c32 = 0; c32 < TILE / 32; ++c32) {
                    float v[32];
                    tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * TILE + 32 * c32), v);
                    // the buffer is free once the previous slice's bulk write has read it
                    if (lane == 0) bulk_wait_read();
                    __syncwarp();
                    // lane = row of the slice; 16-byte chunk c of the row sits at c ^ (row % 8)
                    float4 *dst = reinterpret_cast<float4 *>(ebuf + lane * 128);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[c ^ (lane & 7)] = make_float4(p.alpha * v[4 * c], p.alpha * v[4 * c + 1],
                                                          p.alpha * v[4 * c + 2], p.alpha * v[4 * c + 3]);
                    // generic-proxy writes must be visible to the bulk copy's async proxy
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    const int x = tj * TILE + 32 * c32;
                    if (lane == 0 && x < p.N && row_base < p.M) {
                        if (rd) tma_add_2d(&cmap, ebuf, x, row_base);
                        else tma_store_2d(&cmap, ebuf, x, row_base);
                        bulk_commit();
                    }
                }
            } else {
                // a bulk write of an earlier tile may still be reading the shared buffer
                if (lane == 0) bulk_wait_read();
                __syncwarp();
#pragma unroll 1
                for (int c32 = 0; c32 < TILE / 32; ++c32) {
                    float v[32];
                    if (has_acc) {
                        tmem_ld32(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * TILE + 32 * c32), v);
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = 0.f;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i) stage[lane * 33 + i] = v[i];
                    __syncwarp();
                    const int col = tj * TILE + 32 * c32 + lane;
#pragma unroll
                    for (int r = 0; r < 32; ++r) {
                        const int row = row_base + r;
                        if (row >= p.M || col >= p.N || (p.c_upper && col < row)) continue;
                        const float o = p.alpha * stage[r * 33 + lane];
                        p.C[(long long)row * p.ldc + col] = rd ? fmaf(p.beta, cin[r], o) : o;
                    }
                    __syncwarp();
                    if (rd && c32 + 1 < TILE / 32) epi_load_c(p, row_base, col + 32, cin);
                }
            }
            if (has_acc) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
                ++ch;
            }
        }
        // every bulk write is complete before the CTA (and its shared memory) goes away
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------

// 2D fp32 tensor map over a row-major matrix of `rows` x `cols` (row pitch ld floats) whose
// contiguous index is `cols`; box = box_cols (contiguous) x box_rows.
// mn_major selects the 32-byte-atom variant of the 128-byte swizzle that MN-major tf32
// operands need; K-major operands use the plain 128-byte swizzle.
inline bool make_map_f32(CUtensorMap *map, const float *ptr, long long rows, long long cols,
                         long long ld, int box_cols, int box_rows, bool mn_major) {
    tc::EncodeTiledFn enc = tc::encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 4};
    const cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float *>(ptr), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               mn_major ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// True when the tensor-core path can take this product: 16-byte aligned bases and pitches.
inline bool tc_eligible(const void *A, long long lda, const void *B, long long ldb) {
    return ((reinterpret_cast<uintptr_t>(A) | reinterpret_cast<uintptr_t>(B)) & 15u) == 0 &&
           lda % 4 == 0 && ldb % 4 == 0;
}

}  // namespace tcg
}  // namespace gptq

namespace gptq {

// C = alpha op(A) op(B) + beta C in fp32 accuracy: tcgen05 (tf32 x 3) when the shapes and
// alignments allow it, the SIMT kernel otherwise (small or unaligned products, or when
// GPTQ_FORCE_SIMT_GEMM is set).
inline int gemm_f32(const GemmArgs<float, float> &g, cudaStream_t s) {
    if (g.M <= 0 || g.N <= 0) return GPTQ_OK;
    static const bool force_simt = std::getenv("GPTQ_FORCE_SIMT_GEMM") != nullptr;
    const bool small = (long long)g.M * g.N < 128LL * 256 || g.K < 64;
    // split operands on the SIMT path: C = alpha (A_hi + A_lo)(B_hi + B_lo) + beta C as one
    // product per pair of parts
    auto simt = [&]() -> int {
        GemmArgs<float, float> h = g;
        h.a_lo = nullptr;
        h.b_lo = nullptr;
        if (g.b_lo && g.b_full) {
            h.B = g.b_full;
            h.ldb = g.ldb_full;
        }
        if (!g.a_lo && (!g.b_lo || g.b_full)) return gemm_simt(h, s);
        const float *as[2] = {g.A, g.a_lo}, *bs[2] = {h.B, g.b_full ? nullptr : g.b_lo};
        bool first = true;
        for (int i = 0; i < 2; ++i) {
            for (int j = 0; j < 2; ++j) {
                if (!as[i] || !bs[j]) continue;
                h.A = as[i];
                h.B = bs[j];
                h.beta = first ? g.beta : 1.f;
                first = false;
                if (int st = gemm_simt(h, s)) return st;
            }
        }
        return GPTQ_OK;
    };
    if (small || !tcg::tc_eligible(g.A, g.lda, g.B, g.ldb) ||
        (g.a_lo && !tcg::tc_eligible(g.a_lo, g.lda, g.B, g.ldb)) ||
        (g.b_lo && !tcg::tc_eligible(g.A, g.lda, g.b_lo, g.ldb)) ||
        (reinterpret_cast<uintptr_t>(g.C) & 3u) || force_simt)
        return simt();
    tcg::TcGemmParams p;
    p.M = g.M; p.N = g.N; p.K = g.K;
    p.C = g.C; p.ldc = g.ldc;
    p.alpha = g.alpha; p.beta = g.beta;
    p.a_mn = g.ta ? 1 : 0;
    p.b_mn = g.tb ? 0 : 1;
    p.c_upper = g.c_upper; p.a_upper = g.a_upper; p.a_lower = g.a_lower;
    p.b_upper = g.b_upper; p.b_lower = g.b_lower;
    p.tiles_m = ceil_div(g.M, tcg::TILE);
    p.tiles_n = ceil_div(g.N, tcg::TILE);
    static const long long wait_limit = tc::env_ll("GPTQ_WAIT_LIMIT_CYCLES", 4000000000LL);
    p.wait_limit = wait_limit;
    p.skip = g.skip;
    CUtensorMap am, bm, cm;
    const bool ok_a = p.a_mn ? tcg::make_map_f32(&am, g.A, g.K, g.M, g.lda, 32, 32, true)
                             : tcg::make_map_f32(&am, g.A, g.M, g.K, g.lda, 32, tcg::TILE, false);
    const bool ok_b = p.b_mn ? tcg::make_map_f32(&bm, g.B, g.K, g.N, g.ldb, 32, 32, true)
                             : tcg::make_map_f32(&bm, g.B, g.N, g.K, g.ldb, 32, tcg::TILE, false);
    CUtensorMap alm;
    p.a_split = g.a_lo ? 1 : 0;
    const bool ok_al = !g.a_lo ||
        (p.a_mn ? tcg::make_map_f32(&alm, g.a_lo, g.K, g.M, g.lda, 32, 32, true)
                : tcg::make_map_f32(&alm, g.a_lo, g.M, g.K, g.lda, 32, tcg::TILE, false));
    CUtensorMap blm;
    p.b_split = g.b_lo ? 1 : 0;
    const bool ok_bl = !g.b_lo ||
        (p.b_mn ? tcg::make_map_f32(&blm, g.b_lo, g.K, g.N, g.ldb, 32, 32, true)
                : tcg::make_map_f32(&blm, g.b_lo, g.N, g.K, g.ldb, 32, tcg::TILE, false));
    if (!ok_a || !ok_b || !ok_al || !ok_bl) return simt();
    if (!g.a_lo) alm = am;   // not read
    if (!g.b_lo) blm = bm;   // not read
    // C through a tensor map when beta is 0 or 1 and C's base and pitch allow it
    static const bool rmw_only = std::getenv("GPTQ_GEMM_RMW_EPILOGUE") != nullptr;
    p.c_tma = !rmw_only && (g.beta == 0.f || g.beta == 1.f) &&
              (reinterpret_cast<uintptr_t>(g.C) & 15u) == 0 && g.ldc % 4 == 0 &&
              tcg::make_map_f32(&cm, g.C, g.M, g.N, g.ldc, 32, 32, false);
    if (!p.c_tma) cm = am;   // not read
    const int sms = device_sm_count();
    const int tiles = tcg::num_tiles(p);
    int grid = tiles < sms ? tiles : sms;
    if (g.max_ctas > 0 && grid > g.max_ctas) grid = g.max_ctas;
    GPTQ_SMEM_LIMIT(tcg::gemm_tc_kernel, tcg::SMEM_BYTES);
    KtSpan span(s, g.skip != nullptr);
    const int st = launch_kernel(tcg::gemm_tc_kernel, dim3(grid), dim3(tcg::THREADS), tcg::SMEM_BYTES,
                                 s, g.pdl != 0, am, bm, cm, alm, blm, p);
    span.done(KT_TC, g);
    return st;
}

}  // namespace gptq
