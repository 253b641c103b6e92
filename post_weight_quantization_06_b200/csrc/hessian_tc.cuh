// H += 2 X^T X on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// GPTQ (encyclopedia article), "Technical approach": the quantizer is driven by the Hessian
// of the layer-wise squared error, 2 X^T X for the calibration matrix X (tokens x features).
//
// Shape of the computation: X is k x n row-major (features contiguous). H's upper triangle
// is cut into 256 x 256 tiles (I, J), I <= J, each computed by a CTA pair (a cluster of two,
// tcgen05 cta_group::2): D[i][j] = sum_t X[t][256 I + i] X[t][256 J + j], i.e. A = X[:, I-slab]^T
// and B = X[:, J-slab]^T, both "MN-major" in UMMA terms (the feature index is the contiguous
// one, the token index K is strided). CTA r of the pair holds features 256 I + 128 r .. of A
// and 256 J + 128 r .. of B; the leader's 256 x 256 x 16 MMAs read both CTAs' shared memory
// and leave rows 128 r .. of D in CTA r's TMEM. Per SM this moves two thirds of the operand
// lines of a one-CTA 128 x 256 tile for the same MMA work; the TMA line rate, not HBM or the
// tensor pipe, is what bounds the one-CTA form. TMA brings 64-token x 64-feature boxes with
// the 128-byte swizzle, which is the canonical MN-major SW128 operand layout.
//
// Work units: tile t runs as one unit, except the tiles left over after the last full round
// of pairs, which are cut into token parts so that the last round is full too; a part's
// partial sum goes to a full 256 x 256 block below H's diagonal (free until the final
// mirror) and a small kernel adds the parts into H in part order. No pair waits for another.
//
// Warp roles (320 threads per CTA, one CTA per SM):
//   warp 0      TMA producer (both CTAs): 6-stage ring of this CTA's {A, B} halves (32 KB per
//               stage; a diagonal tile loads B only and uses it for both operands); the loads
//               complete on the leader's full barrier, armed by the leader for both CTAs
//   warp 1      TMEM allocation (both CTAs) and, in the leader, the MMA issuer (one thread):
//               4 x tcgen05.mma (256 x 256 x 16, bf16 in, fp32 accumulate) per stage
//   warps 2-9   epilogue (both CTAs): lane quarter (warp % 4) x column half -> 32 rows x 128
//               columns of this CTA's 128 x 256 accumulator
//
// Precision: the tensor cores accumulate each chunk of 1024 tokens afresh in one of two TMEM
// accumulators (double buffered); the epilogue adds 16 chunk sums in registers and then adds
// that sum into H with fire-and-forget vector reductions (red.global.add), so every element of
// H is a two-level sum (1024 tokens in the tensor core, 16 chunks in registers, k / 16384
// updates of H) rather than a k-token chain. The updates of one element come from one thread
// in program order, so the result is deterministic. (The intrinsic-LoRA Schur step cancels
// H's large eigenvalues down to lambda and needs this accuracy.)
//
// Every mbarrier wait is bounded (clock64); a wait that runs out records GPTQ_ERR_TIMEOUT
// with its site, sets the CTA's abort flag, and all roles leave their loops (the other CTA of
// the pair runs into its own bounded waits); both CTAs then meet at the closing cluster
// barrier and the TMEM is freed.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace gptq {
namespace tc {

constexpr int TILE = 128;          // rows of one CTA's slab; also the tile of tile_coords
constexpr int PAIR_TILE = 256;     // output tile of a CTA pair: 256 x 256
constexpr int BK = 64;             // tokens per pipeline stage
constexpr int STAGES = 6;
constexpr int CHUNK_STAGES = 16;   // 1024 tokens per TMEM partial sum
constexpr int FLUSH_CHUNKS = 16;   // chunk sums added in registers before an update of H
constexpr int BOX_BYTES = 64 * BK * 2;       // one 64-feature x 64-token bf16 box: 8 KB
constexpr int HALF_BYTES = 2 * BOX_BYTES;    // 128 features: 16 KB
constexpr int STAGE_BYTES = 2 * HALF_BYTES;  // this CTA's halves of A and B
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 32 * (2 + EPI_WARPS);
constexpr int TMEM_COLS = 2 * PAIR_TILE;     // two 128-lane x 256-column accumulators
// Each epilogue thread sums 128 columns of its TMEM lane: the first ACC_REGS in registers,
// the rest in shared memory (column-major over the 256 epilogue threads), which keeps the
// kernel within the 168 registers a thread can have with 10 warps per SM and off the
// local-memory spill path.
constexpr int ACC_REGS = 96;
constexpr int ACC_SMEM = 128 - ACC_REGS;
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256 +
                              sizeof(float) * (size_t)ACC_SMEM * EPI_THREADS;
static_assert(SMEM_BYTES <= 232448, "fits the 227 KB of shared memory a CTA may use");

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both MN-major, M = N = 256 (the
// pair's shape: each CTA supplies 128 rows of A and 128 columns of B and receives 128 rows
// of D in its own TMEM).
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                           ((uint32_t)(PAIR_TILE >> 3) << 17) |
                           ((uint32_t)(PAIR_TILE >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// Bounded wait for the phase with the given parity; false if `limit` cycles pass first.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, long long limit) {
    const uint32_t addr = smem_u32(bar);
    const long long t0 = clock64();
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(addr), "r"(parity)
            : "memory");
        if (ok) return true;
        if (clock64() - t0 > limit) return false;
    }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// ---- CTA-pair (cta_group::2) forms, used by the Hessian kernel only: every tcgen05
// instruction of a kernel names the same CTA group.
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// shared::cluster address of `p` (a shared variable of this CTA) in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(const void *p, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
    return a;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on an mbarrier that may
// sit in the peer CTA of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint32_t bar_cluster,
                                                 void *dst, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst)),
                 "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
__device__ __forceinline__ void mma_bf16_pair(uint32_t dtmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(dtmem),
        "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate));
}
// Arrive (once) on the mbarrier at `bar`'s offset in every CTA of `mask` when this thread's
// prior MMAs complete.
__device__ __forceinline__ void mma_commit_pair(uint64_t *bar, uint16_t mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(mask)
        : "memory");
}
__device__ __forceinline__ void red_add_v4(float *p, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}
__device__ __forceinline__ void red_add(float *p, float a) {
    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(a) : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// 16 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: MN-major operand, 128-byte swizzle. LBO = byte distance
// between the two 64-feature halves of the operand, SBO = between 8-token groups.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((BOX_BYTES >> 4) & 0x3FFFu) << 16;  // LBO: next 64 features
    d |= (uint64_t)((1024 >> 4) & 0x3FFFu) << 32;       // SBO: next 8 tokens
    d |= (uint64_t)1 << 46;                              // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                              // 128-byte swizzle
    return d;
}

// Upper-triangle tile t (row-major over I <= J) of a T x T tile grid.
__device__ __forceinline__ void tile_coords(int t, int T, int &I, int &J) {
    int i = 0;
    while (t >= T - i) { t -= T - i; ++i; }
    I = i;
    J = i + t;
}

struct HessianParams {
    float *H;
    int n;
    long long k;
    int T2;          // ceil(n / 256): pair tiles per side
    int tiles;       // T2 (T2 + 1) / 2 upper-triangle pair tiles
    int whole;       // tiles 0 .. whole-1 run as one unit each
    int tail_parts;  // tiles whole .. tiles-1 run as tail_parts token parts each
    int units;       // whole + (tiles - whole) * tail_parts
    int full_blocks; // floor(n / 256): lower-triangle 256-blocks usable as scratch
    long long wait_limit;
    int stall;       // test hook: epilogue waits on a barrier nothing signals
};

// Unit u -> pair tile t, token chunks [c0, c1), and for a tail part its scratch slot.
__device__ __forceinline__ void hess_unit(const HessianParams &p, int nch, int u, int &t, int &c0,
                                          int &c1, int &slot) {
    if (u < p.whole) {
        t = u;
        c0 = 0;
        c1 = nch;
        slot = -1;
    } else {
        const int j = u - p.whole;
        const int part = j % p.tail_parts;
        t = p.whole + j / p.tail_parts;
        c0 = part * nch / p.tail_parts;
        c1 = (part + 1) * nch / p.tail_parts;
        slot = j;
    }
}

// Scratch slot s: the s-th full 256 x 256 block strictly below the diagonal of H (row-major
// over block rows 1 .. full_blocks-1), free until the final mirror.
__device__ __forceinline__ float *hess_slot(const HessianParams &p, int s) {
    int bi = 1;
    while (s >= bi) { s -= bi; ++bi; }
    return p.H + (long long)bi * PAIR_TILE * p.n + (long long)s * PAIR_TILE;
}

// One CTA pair (cluster of 2; rank 0 leads) per 256 x 256 tile of H's upper triangle. Rank r
// loads features 256 I + 128 r .. (its half of A) and 256 J + 128 r .. (its half of B) for
// each 64-token stage; the leader's single MMA thread issues 256 x 256 x 16 MMAs that read
// both CTAs' shared memory and write 128 rows into each CTA's TMEM.
//   Barriers: the leader's full[s] counts its own arrive (with both CTAs' bytes) and both
// CTAs' TMA bytes; the leader's commits arrive on empty[s] and acc_full[b] of both CTAs; the
// epilogue warps of both CTAs arrive on the leader's acc_empty[b].
__global__ void __launch_bounds__(THREADS, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap xmap, HessianParams p) {
    extern __shared__ __align__(1024) unsigned char smraw[];
    unsigned char *base = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smraw) + 1023) & ~uintptr_t(1023));
    unsigned char *stages = base;
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                    // STAGES (used in the leader)
    uint64_t *empty = bars + STAGES;          // STAGES
    uint64_t *acc_full = bars + 2 * STAGES;   // 2
    uint64_t *acc_empty = acc_full + 2;       // 2 (used in the leader)
    uint64_t *mma_done = acc_empty + 2;       // 1
    uint64_t *never = mma_done + 1;           // 1 (test hook)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(never + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const long long nk = (p.k + BK - 1) / BK;
    const int nch = (int)((nk + CHUNK_STAGES - 1) / CHUNK_STAGES);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 2 * EPI_WARPS);
        }
        mbar_init(mma_done, 1);
        mbar_init(never, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers exist before any remote arrive or TMA
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            long long it = 0;
            for (int u = pair; u < p.units && !*abort_flag; u += npairs) {
                int t, c0, c1, slot, I, J;
                hess_unit(p, nch, u, t, c0, c1, slot);
                tile_coords(t, p.T2, I, J);
                const bool diag = I == J;  // this CTA's A half equals its B half
                const long long s0 = (long long)c0 * CHUNK_STAGES;
                const long long s1 = (long long)c1 * CHUNK_STAGES < nk ? (long long)c1 * CHUNK_STAGES : nk;
                for (long long ks = s0; ks < s1; ++ks, ++it) {
                    const int st = (int)(it % STAGES);
                    const uint32_t par = (uint32_t)((it / STAGES) & 1) ^ 1u;
                    if (*abort_flag) break;
                    if (!mbar_wait(&empty[st], par, p.wait_limit)) {
                        report(GPTQ_ERR_TIMEOUT, 1);
                        *abort_flag = 1;
                        break;
                    }
                    unsigned char *sA = stages + st * STAGE_BYTES;
                    unsigned char *sB = sA + HALF_BYTES;
                    if (rank == 0) mbar_expect_tx(&full[st], 2u * (diag ? HALF_BYTES : STAGE_BYTES));
                    const uint32_t fb = map_to_rank(&full[st], 0);
                    const int y = (int)(ks * BK);
                    const int xa = I * PAIR_TILE + TILE * (int)rank, xb = J * PAIR_TILE + TILE * (int)rank;
                    if (!diag) {
                        tma_load_2d_pair(&xmap, fb, sA, xa, y);
                        tma_load_2d_pair(&xmap, fb, sA + BOX_BYTES, xa + 64, y);
                    }
                    tma_load_2d_pair(&xmap, fb, sB, xb, y);
                    tma_load_2d_pair(&xmap, fb, sB + BOX_BYTES, xb + 64, y);
                }
            }
            if (*abort_flag) {
                // copies in flight land within microseconds; give them time before the
                // shared memory goes away (their barrier may sit in the other CTA)
                const long long t0 = clock64();
                while (clock64() - t0 < 2000000) { }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader only) ----------------
        if (rank == 0 && lane == 0) {
            long long it = 0, ch = 0;
            for (int u = pair; u < p.units && !*abort_flag; u += npairs) {
                int t, c0, c1, slot, I, J;
                hess_unit(p, nch, u, t, c0, c1, slot);
                tile_coords(t, p.T2, I, J);
                const bool diag = I == J;
                for (int c = c0; c < c1 && !*abort_flag; ++c, ++ch) {
                    const int b = (int)(ch & 1);
                    if (!mbar_wait(&acc_empty[b], (uint32_t)((ch >> 1) & 1) ^ 1u, p.wait_limit)) {
                        report(GPTQ_ERR_TIMEOUT, 2);
                        *abort_flag = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dt = tmem + (uint32_t)(b * PAIR_TILE);
                    const long long s0 = (long long)c * CHUNK_STAGES;
                    const long long s1 = s0 + CHUNK_STAGES < nk ? s0 + CHUNK_STAGES : nk;
                    for (long long ks = s0; ks < s1; ++ks, ++it) {
                        const int st = (int)(it % STAGES);
                        if (!mbar_wait(&full[st], (uint32_t)((it / STAGES) & 1), p.wait_limit)) {
                            report(GPTQ_ERR_TIMEOUT, 3);
                            *abort_flag = 1;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t b0 = smem_u32(stages + st * STAGE_BYTES) + HALF_BYTES;
                        const uint32_t a0 = diag ? b0 : b0 - HALF_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint32_t off = (uint32_t)kk * 16u * 128u;  // 16 tokens x 128 B
                            mma_bf16_pair(dt, desc_mn_sw128(a0 + off), desc_mn_sw128(b0 + off),
                                          (ks > s0 || kk > 0) ? 1u : 0u);
                        }
                        mma_commit_pair(&empty[st], 0x3);
                    }
                    mma_commit_pair(&acc_full[b], 0x3);
                }
            }
            // all MMAs of this thread complete before the pair's TMEM is released
            mma_commit_pair(mma_done, 0x1);
            mbar_wait(mma_done, 0, p.wait_limit);
        }
    } else {
        // ---------------- epilogue (both CTAs) ----------------
        const int e = warp - 2;
        const int q = warp & 3;         // TMEM lane quarter this warp may access
        const int h = e >> 2;           // column half
        float acc[ACC_REGS];
        float *acc_sm = reinterpret_cast<float *>(base + STAGES * STAGE_BYTES + 256) +
                        (threadIdx.x - 64);  // column j at acc_sm[j * EPI_THREADS]
        int ch = 0;
        if (p.stall) {
            if (!mbar_wait(never, 0, p.wait_limit)) {
                if (lane == 0) report(GPTQ_ERR_TIMEOUT, 4);
                *abort_flag = 1;
            }
        }
        // running sum of column c of this thread (c compile-time after unrolling)
#define HESS_ACC(c) (*((c) < ACC_REGS ? &acc[(c) < ACC_REGS ? (c) : 0] \
                                       : &acc_sm[((c) < ACC_REGS ? 0 : (c) - ACC_REGS) * EPI_THREADS]))
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(128 * h);
        const uint32_t rel0 = map_to_rank(&acc_empty[0], 0), rel1 = map_to_rank(&acc_empty[1], 0);
        for (int u = pair; u < p.units && !*abort_flag; u += npairs) {
            int t, c0, c1, slot;
            hess_unit(p, nch, u, t, c0, c1, slot);
#pragma unroll
            for (int c = 0; c < 128; ++c) HESS_ACC(c) = 0.f;
            bool first = true;
            int c = c0;
            for (; c < c1; ++c, ++ch) {
                const int b = ch & 1;
                if (!mbar_wait(&acc_full[b], (uint32_t)((ch >> 1) & 1), p.wait_limit)) {
                    if (lane == 0) report(GPTQ_ERR_TIMEOUT, 5);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t ta = tq + (uint32_t)(b * PAIR_TILE);
#pragma unroll
                for (int part8 = 0; part8 < 16; ++part8) {
                    float v[8];
                    tmem_ld8(ta + 8 * part8, v);
#pragma unroll
                    for (int i = 0; i < 8; ++i) HESS_ACC(8 * part8 + i) += v[i];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(b ? rel1 : rel0);
                if ((c - c0 + 1) % FLUSH_CHUNKS != 0 && c + 1 != c1) continue;
                // ---- flush 2 acc: into H (upper triangle) or into the part's scratch slot ----
                int I, J;
                tile_coords(t, p.T2, I, J);
                const int rloc = TILE * (int)rank + 32 * q + lane;  // row within the pair tile
                const int row = I * PAIR_TILE + rloc;
                const int col0 = J * PAIR_TILE + 128 * h;
                if (slot >= 0) {
                    // scratch rows are full; store the first flush, add the later ones
                    float *Sr = hess_slot(p, slot) + (long long)rloc * p.n + 128 * h;
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        float4 v = make_float4(2.f * HESS_ACC(4 * x), 2.f * HESS_ACC(4 * x + 1),
                                               2.f * HESS_ACC(4 * x + 2), 2.f * HESS_ACC(4 * x + 3));
                        if (first) *reinterpret_cast<float4 *>(Sr + 4 * x) = v;
                        else red_add_v4(Sr + 4 * x, v.x, v.y, v.z, v.w);
                    }
                } else if (row < p.n) {
                    float *Hr = p.H + (long long)row * p.n + col0;
                    const int rbase = I * PAIR_TILE + TILE * (int)rank + 32 * q;
                    if (col0 >= rbase + 31 && col0 + 127 < p.n) {
                        // the warp's whole 32 x 128 block is on or above the diagonal
#pragma unroll
                        for (int x = 0; x < 32; ++x)
                            red_add_v4(Hr + 4 * x, 2.f * HESS_ACC(4 * x), 2.f * HESS_ACC(4 * x + 1),
                                       2.f * HESS_ACC(4 * x + 2), 2.f * HESS_ACC(4 * x + 3));
                    } else if (col0 + 127 >= rbase) {
#pragma unroll
                        for (int cc = 0; cc < 128; ++cc) {
                            const int col = col0 + cc;
                            if (col >= row && col < p.n) red_add(Hr + cc, 2.f * HESS_ACC(cc));
                        }
                    }
                }
                first = false;
#pragma unroll
                for (int cc = 0; cc < 128; ++cc) HESS_ACC(cc) = 0.f;
            }
            if (c < c1) break;  // left on an abort
        }
#undef HESS_ACC
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // the peer's TMEM, barriers and shared memory outlive every access
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

// H (upper part of the tail tiles) += the parts' partial sums, in part order.
__global__ void hessian_tail_reduce_kernel(HessianParams p) {
    const int per_tile = PAIR_TILE * PAIR_TILE;
    const long long total = (long long)(p.tiles - p.whole) * per_tile;
    for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int tt = (int)(idx / per_tile), e = (int)(idx % per_tile);
        const int rl = e / PAIR_TILE, cl = e % PAIR_TILE;
        int I, J;
        tile_coords(p.whole + tt, p.T2, I, J);
        const int row = I * PAIR_TILE + rl, col = J * PAIR_TILE + cl;
        if (row >= p.n || col >= p.n || col < row) continue;
        float acc = p.H[(long long)row * p.n + col];
        for (int part = 0; part < p.tail_parts; ++part)
            acc += hess_slot(p, tt * p.tail_parts + part)[(long long)rl * p.n + cl];
        p.H[(long long)row * p.n + col] = acc;
    }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

inline long long env_ll(const char *name, long long dflt) {
    const char *v = getenv(name);
    return v && *v ? atoll(v) : dflt;
}

// H (upper triangle) += 2 X^T X; the lower triangle is overwritten (scratch of the tail
// parts, then the mirror of the upper one, done by the caller). X: k x n bf16 row-major,
// 16-byte aligned, n % 8 == 0.
inline int hessian_tc(float *H, const __nv_bfloat16 *X, long long k, int n, cudaStream_t s) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return GPTQ_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)k};
    const cuuint64_t strides[1] = {(cuuint64_t)n * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)BK};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(X), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return GPTQ_ERR_CUDA;
    GPTQ_SMEM_LIMIT(hessian_tc_kernel, SMEM_BYTES);
    HessianParams p;
    p.H = H;
    p.n = n;
    p.k = k;
    p.T2 = (n + PAIR_TILE - 1) / PAIR_TILE;
    p.tiles = p.T2 * (p.T2 + 1) / 2;
    p.full_blocks = n / PAIR_TILE;
    const long long nk = (k + BK - 1) / BK;
    const int nch = (int)((nk + CHUNK_STAGES - 1) / CHUNK_STAGES);
    // pairs resident at once (a pair never waits for another, so fewer is only slower)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const int sms = device_sm_count();
    cfg.gridDim = dim3(2 * (sms / 2));
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, hessian_tc_kernel, &cfg) != cudaSuccess ||
        clusters < 1)
        clusters = sms / 2;
    // whole tiles fill full rounds; the tail tiles are cut into token parts that fill the
    // last round, their partial sums kept in full 256-blocks below the diagonal
    const int rounds = p.tiles / clusters;
    const int tail = p.tiles - rounds * clusters;
    int parts = 1;
    if (tail > 0 && rounds > 0) {
        const int lower = p.full_blocks * (p.full_blocks - 1) / 2;
        parts = clusters / tail;
        if (parts > nch) parts = nch;
        if (parts * tail > lower) parts = lower / tail;
        if (parts < 2) parts = 1;
    }
    const long long forced = env_ll("GPTQ_HESSIAN_TAIL_PARTS", 0);
    if (forced == 1) parts = 1;
    p.whole = parts > 1 ? rounds * clusters : p.tiles;
    p.tail_parts = parts > 1 ? parts : 1;
    p.units = p.whole + (p.tiles - p.whole) * p.tail_parts;
    // a wait longer than ~2 s at the 1.9 GHz clock means a lost signal, not a slow kernel
    p.wait_limit = env_ll("GPTQ_WAIT_LIMIT_CYCLES", 4000000000LL);
    p.stall = (int)env_ll("GPTQ_TEST_STALL", 0);
    const int pairs = p.units < clusters ? p.units : clusters;
    cfg.gridDim = dim3(2 * pairs);
    if (cudaLaunchKernelEx(&cfg, hessian_tc_kernel, map, p) != cudaSuccess) return launch_status();
    if (int st = launch_status()) return st;
    if (p.whole < p.tiles) {
        hessian_tail_reduce_kernel<<<sms * 4, 256, 0, s>>>(p);
        if (int st = launch_status()) return st;
    }
    return GPTQ_OK;
}

}  // namespace tc
}  // namespace gptq
