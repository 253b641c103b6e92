/*
 * gptq.h — C ABI of the B200 (sm_100a) GPTQ layer-quantization library (libgptq.so).
 *
 * The library runs the GPTQ layer-wise quantization pass and its
 * GPTQ-intrinsic-LoRA variant on one GPU:
 *
 *   gptq_hessian_accumulate   H += 2 X^T X over one chunk of calibration tokens
 *   gptq_prepare_hinv         lambda = lambda_rel * mean(diag H); U upper with (H + lambda I)^-1 = U^T U
 *   gptq_quantize_layer       column sweep of W onto per-group min-max grids with error feedback
 *   gptq_il_quantize_layer    the same pass on the augmented calibration [X, X V_r]; returns Q, L = V_r, R
 *   gptq_il_refine            OLrC + Bid-Up refinement rounds on a quantized layer: new L, R, codes
 *   gptq_quantize_lowrank     L and R stored at low precision (4-bit L, 8-bit R) on min-max grids
 *   gptq_2d_round             two-sided adaptive rounding of a real matrix to integers (GPTQ-2D)
 *   gptq_quantize_layer_reduced  GPTQ after LLL reduction of the data lattice (per-channel grid)
 *   gptq_set_flags            synchronous status returns and debug synchronisation (see below)
 *   gptq_kernel_times         device time and algorithmic work of the GEMM launches (diagnostic)
 *
 * Conventions shared by every entry point
 *   - Orientation: W is m x n row-major (m output rows, n input columns: one neuron per row);
 *     X is k x n row-major (k calibration tokens). The pages write the layer as XW with W
 *     stored in x out; this is its transpose. Columns are swept j = 0 .. n-1.
 *   - Every pointer argument named as "device" must point to device memory of the current
 *     device, owned by the caller; the library never allocates or frees device memory.
 *     Scratch memory is passed in as `workspace` (size from gptq_workspace_size).
 *   - Calls only enqueue work on `stream` (a cudaStream_t; NULL = the legacy default stream)
 *     and return without synchronising. Argument errors are detected on the host and
 *     returned at once (GPTQ_ERR_ARG / GPTQ_ERR_WORKSPACE); nothing is enqueued then.
 *     Errors the device finds (a non-positive pivot, non-finite data, a timed-out wait)
 *     are recorded in a sticky per-device status word: the first error wins and later
 *     calls keep running on whatever data they get. Read and clear it with
 *     gptq_sync_status(). A launch failure reported by the CUDA runtime is returned as
 *     GPTQ_ERR_CUDA.
 *   - There is no CPU fallback: every step runs in this library's CUDA kernels.
 *   - Not thread-safe per device for overlapping calls that share a workspace.
 */
#ifndef GPTQ_H
#define GPTQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GPTQ_API __attribute__((visibility("default")))
#else
#define GPTQ_API
#endif

typedef struct CUstream_st *gptq_stream_t; /* same type as cudaStream_t */

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_ARG = -1,        /* bad pointer, size or option (host-side check) */
    GPTQ_ERR_NOT_PD = -2,     /* a pivot <= 0 in the factorization (info: the column) */
    GPTQ_ERR_NONFINITE = -3,  /* NaN or Inf in W or in diag(H) (info: the flat index) */
    GPTQ_ERR_TIMEOUT = -4,    /* a bounded device-side wait gave up (info: the site) */
    GPTQ_ERR_CUDA = -5,       /* the CUDA runtime refused a launch (see cudaGetLastError) */
    GPTQ_ERR_WORKSPACE = -6,  /* workspace pointer NULL, misaligned or too small */
    GPTQ_ERR_NOT_CONVERGED = -7 /* the top-r eigenvector iteration hit its cap before its
                                   residual test passed (info: iterations run); the outputs
                                   are those of the last iteration */
} gptq_status;

typedef enum { GPTQ_BF16 = 0, GPTQ_F32 = 1 } gptq_dtype;

typedef enum {
    GPTQ_OP_HESSIAN = 0,
    GPTQ_OP_PREPARE_HINV = 1,
    GPTQ_OP_QUANTIZE = 2,
    GPTQ_OP_IL_QUANTIZE = 3,
    GPTQ_OP_IL_REFINE = 4,
    GPTQ_OP_2D_ROUND = 5,
    GPTQ_OP_REDUCED = 6
} gptq_op;

/* Process-wide behaviour flags (gptq_set_flags; default 0):
 *   GPTQ_FLAG_SYNC_STATUS   every compute entry point synchronises its stream after enqueueing
 *                           and returns the device status word (read and cleared, as
 *                           gptq_sync_status does), so device-found errors are returned by the
 *                           call that caused them.
 *   GPTQ_FLAG_DEBUG_CHECKS  as SYNC_STATUS, after a device-wide synchronise that also surfaces
 *                           errors of the library's side streams (GPTQ_ERR_CUDA).
 *   GPTQ_FLAG_IL_FP64       accepted for compatibility: the intrinsic-LoRA path always forms its
 *                           cancelling products (Gram matrices, Schur complement) with fp64
 *                           accumulation.
 *   GPTQ_FLAG_KERNEL_TIMES  note the device time of every fp32 GEMM launch (gptq_kernel_times). */
typedef enum {
    GPTQ_FLAG_SYNC_STATUS = 1u,
    GPTQ_FLAG_DEBUG_CHECKS = 2u,
    GPTQ_FLAG_IL_FP64 = 4u,
    GPTQ_FLAG_KERNEL_TIMES = 8u
} gptq_flag;

GPTQ_API void gptq_set_flags(unsigned flags);
GPTQ_API unsigned gptq_get_flags(void);

/* Bytes of device workspace the entry point `op` needs for these sizes (0 if none).
 * m, n: layer shape; r: intrinsic-LoRA rank (IL only, else 0); block_size: B.
 * The workspace must be 256-byte aligned. Returns 0 for an unknown op. */
GPTQ_API size_t gptq_workspace_size(int op, int64_t m, int64_t n, int r, int block_size);

/* Human-readable name of a gptq_status value (static string, never NULL). */
GPTQ_API const char *gptq_status_string(int status);

/* Waits for `stream`, then returns the device status word of the current device
 * (GPTQ_OK if no device-side error was recorded) and clears it. If `info` is not
 * NULL it receives the error's detail (column / index / site; 0 if none). */
GPTQ_API int gptq_sync_status(gptq_stream_t stream, int64_t *info);

/* Number of CUDA kernels this library has launched in this process so far (all devices).
 * A diagnostic for tracing and benchmarking: the difference of two readings counts the
 * kernels a span of calls launched. Library-internal memsets are not counted. */
GPTQ_API uint64_t gptq_launch_count(void);

/* Device time of the library's fp32 GEMM launches, a benchmarking diagnostic.
 * While GPTQ_FLAG_KERNEL_TIMES is set, every launch of the fp32 GEMM (the tf32 x 3 tensor-core
 * kernel and the SIMT kernel) is bracketed by two CUDA events on its stream and noted with the
 * stage that issued it and its algorithmic work. The events also order launches that would
 * otherwise overlap a predecessor's tail, so a pass run with the flag is a little slower.
 *
 * gptq_kernel_times waits for every noted launch to finish, writes the totals of the first
 * n_out classes to out[0 .. n_out) (class index = stage * 2 + path; path 0 = tensor core,
 * 1 = SIMT; stage = gptq_kt_stage), clears the record, and returns the number of classes
 * (GPTQ_KT_NCLASSES) or GPTQ_ERR_ARG (out NULL with n_out > 0, n_out < 0) or GPTQ_ERR_CUDA.
 * Records of launches on a device other than the current one are read as well.
 *   launches  number of launches
 *   ms        sum of their event-to-event durations (a launch that waits for SMs held by
 *             another stream's kernel counts that wait)
 *   flops     2 x the multiply-adds with both factors structurally nonzero, over the written
 *             entries of C (triangular operands and outputs counted exactly)
 *   bytes     each structurally nonzero operand element read once, each written element of C
 *             stored once and loaded once when beta != 0 */
typedef enum {
    GPTQ_KT_OTHER = 0,
    GPTQ_KT_FACTOR = 1, /* blocked UL factor and inverse (gptq_prepare_hinv, the 2D factors) */
    GPTQ_KT_SWEEP = 2,  /* lazy trailing updates of the column sweep */
    GPTQ_KT_IL = 3,     /* intrinsic-LoRA products (Gram, subspace iteration, Schur complement) */
    GPTQ_KT_REFINE = 4, /* OLrC + Bid-Up products */
    GPTQ_KT_2D = 5,     /* two-sided rounding (its own products) */
    GPTQ_KT_NSTAGES = 6
} gptq_kt_stage;
#define GPTQ_KT_NCLASSES 12

typedef struct {
    int64_t launches;
    double ms;
    double flops;
    double bytes;
} gptq_kernel_time;

GPTQ_API int gptq_kernel_times(gptq_kernel_time *out, int n_out);

/*
 * H += 2 X^T X.
 * GPTQ (encyclopedia article), "Technical approach": the quantizer is driven by the
 * Hessian of the layer-wise squared error ||XW - XQ||^2, which is 2 X^T X.
 *   H       device, n x n fp32 row-major, caller-owned; accumulated into (zero it before
 *           the first chunk). Only the upper triangle (diagonal included) is read; the
 *           strictly lower one may serve as scratch during the call. On return both
 *           triangles hold the symmetric sum.
 *   X       device, k x n row-major calibration chunk; x_dtype GPTQ_BF16 or GPTQ_F32.
 *           The base address must be 16-byte aligned; for GPTQ_BF16, n % 8 == 0. bf16 X runs
 *           on the bf16 tensor cores with fp32 accumulation; fp32 X on the fp32-accurate
 *           tensor-core product (tf32 x 3: each operand split into two tf32 parts, three
 *           products; error ~2^-22 of |x||y| per product) when n % 4 == 0 and n x n is large
 *           enough, else on an fp32 SIMT kernel.
 *   k, n    k >= 0 tokens (k == 0 is a no-op), 1 <= n <= 65536 features.
 * Call it once per chunk of tokens; chunks are additive and may be of any length.
 */
GPTQ_API int gptq_hessian_accumulate(float *H, const void *X, int x_dtype, int64_t k, int64_t n,
                            gptq_stream_t stream);

/*
 * lambda = lambda_rel * mean(diag H);  U upper triangular with (H + lambda I)^-1 = U^T U.
 * GPTQ-2D (two-sided adaptive rounding), sections 2 and 4: the error feedback is read
 * from a triangular factor of the inverse Gram matrix; Lattice Geometry of Neural
 * Network Quantization, section 3.1: lambda regularisation keeps the basis independent.
 * Computed as H + lambda I = Ubar Ubar^T (Cholesky from the last column backwards,
 * Ubar upper) followed by U = Ubar^-1: the same U as chol -> inverse -> chol.
 *   H          device, n x n fp32 (the raw 2 X^T X), read only; only the upper triangle
 *              is read.
 *   lambda_rel relative damping (> 0 recommended; >= 0 accepted).
 *   U          device, n x n fp32, written: the upper triangle (diagonal included) holds
 *              U; the strictly lower triangle is left zero.
 *   lambda_out device, one fp32: the absolute lambda used.
 *   workspace  device, >= gptq_workspace_size(GPTQ_OP_PREPARE_HINV, 0, n, 0, 0) bytes.
 * Device errors: GPTQ_ERR_NOT_PD (info = first column with pivot <= 0),
 * GPTQ_ERR_NONFINITE (info = index of a non-finite diagonal entry of H).
 */
GPTQ_API int gptq_prepare_hinv(const float *H, int64_t n, float lambda_rel, float *U,
                      float *lambda_out, void *workspace, size_t ws_bytes,
                      gptq_stream_t stream);

/*
 * Quantize the columns of W one at a time with closed-form error feedback.
 * GPTQ (encyclopedia article), "Technical approach" (column-wise greedy quantization,
 * closed-form compensation of the remaining weights, per-group scales, 2/3/4-bit);
 * GPTQ-2D, section 2 (GPTQ's lazy block update).
 * For each column j: at a group start the grid of each row is taken from the current
 * weights of the group (xmin = min(0, min w), xmax = max(0, max w), a zero range widened
 * to [-1, 1], s = (xmax - xmin)/maxq, z = rint(-xmin/s)); v = w_j/s + z;
 * c = clamp(rint(v), 0, maxq) (round half to even); e = (w_j - s(c - z)) / U_jj;
 * the later columns of the row receive -e * U_{j, j+1:}. Inside a block of
 * `block_size` columns this is done column by column; the columns after the block are
 * updated once per block by W[:, after] -= Err * U[block, after].
 *   W          device, m x n row-major, w_dtype GPTQ_BF16 or GPTQ_F32, read only.
 *   U          device, n x n fp32 upper factor from gptq_prepare_hinv (row-major).
 *   bits       2..8.  group_size: 0 (one group per row) or a divisor of n with
 *              block_size % group_size == 0 or group_size % block_size == 0.
 *   block_size 32, 64 or 128; n % block_size == 0.
 *   codes      device, m x (n*bits/32) uint32 (n*bits % 32 == 0): along each row, code j
 *              occupies bits [j*bits, j*bits + bits) of a little-endian bit stream cut
 *              into 32-bit words, least significant bit first.
 *   scales     device, m x G fp32, G = group_size ? n/group_size : 1.
 *   zeros      device, m x G uint8 zero-points.
 *   loss_out   device, m fp64 or NULL: per row sum_j e_j^2, which equals
 *              (w - w_hat)^T (H + lambda I) (w - w_hat).
 *   workspace  device, >= gptq_workspace_size(GPTQ_OP_QUANTIZE, m, n, 0, block_size).
 * Device errors: GPTQ_ERR_NONFINITE (info = flat index into W of a non-finite weight).
 */
GPTQ_API int gptq_quantize_layer(const void *W, int w_dtype, int64_t m, int64_t n, const float *U,
                        int bits, int group_size, int block_size, uint32_t *codes,
                        float *scales, uint8_t *zeros, double *loss_out, void *workspace,
                        size_t ws_bytes, gptq_stream_t stream);

/*
 * gptq_quantize_layer without a workspace argument and without any allocation.
 * The pages have no counterpart to this entry point: it exists for callers that cannot
 * hand the library device scratch memory, e.g. code running under a memory pool it does
 * not own (a framework allocator that has reserved the device), or code that must not call
 * cudaMalloc because it can synchronize the whole device and stall other work.
 * It runs the same kernels as gptq_quantize_layer, with their scratch (the fp32 working
 * copy of W and the per-panel errors) placed in a file-scope device array of
 * GPTQ_NOALLOC_SCRATCH_BYTES bytes that every device loading the library holds until the
 * process exits. The caller still provides W, U and the outputs, as for
 * gptq_quantize_layer, and the arguments mean the same.
 *   - Limit: the scratch, m * n floats (the working copy) plus
 *     2 * m * max(min(n, 1024), block_size) floats (the errors of one 1024-column outer
 *     block, kept as a tf32 high part and its remainder), each part rounded up to 256 bytes,
 *     must not exceed GPTQ_NOALLOC_SCRATCH_BYTES; e.g. 2048 x 6144 fits (exactly), 2048 x 7680
 *     does not. Larger layers get GPTQ_ERR_ARG and nothing is enqueued. (gptq_quantize_layer's
 *     workspace also holds U's outer-block band split into tf32 pairs, which this entry point
 *     does without: its tensor-core products split U as they load it. Both round the same
 *     way, so the outputs are identical.)
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *     with that device current; make that first call before any stream capture. The address
 *     is tied to the device's current context: a call made after that context was destroyed
 *     and replaced (cudaDeviceReset, or a framework that resets the device) looks it up again
 *     (and must then come before any capture too).
 *   - Every call on a device shares the one array and leaves its contents behind. Calls
 *     whose work overlaps on the GPU (other streams, other host threads) race on it:
 *     serialise them. Nothing in the array needs to start at zero.
 *   - Never calls cudaMalloc, cudaFree or any allocating routine.
 */
#define GPTQ_NOALLOC_SCRATCH_BYTES (64u << 20)
GPTQ_API int gptq_quantize_layer_noalloc(const void *W, int w_dtype, int64_t m, int64_t n,
                                         const float *U, int bits, int group_size,
                                         int block_size, uint32_t *codes, float *scales,
                                         uint8_t *zeros, double *loss_out,
                                         gptq_stream_t stream);

/*
 * GPTQ-intrinsic LoRA: quantize W against the augmented calibration X~ = [X, X V_r].
 * GPTQ-intrinsic LoRA summary, "Method" part 2: V_r (= L) are the top-r right singular
 * vectors of X; the pass runs on W~ = [W, 0] (r extra zero-initialised coordinates per
 * row, placed after the n original ones and never quantized); the extra coordinates
 * absorb the quantization error and end as R; the singular augmented Hessian is factored
 * without a plain Cholesky of it. Here: V_r by subspace iteration on H (a block of
 * p = min(max(r + 32, 2r), 128, n) columns): power steps with fp32-accurate tensor-core
 * products first, then fp64-accumulated iterations, each with a Rayleigh-Ritz step, until
 * every one of the r Ritz pairs (theta, v) has ||H v - theta v|| <= 5e-6 theta (at most 12
 * fp64 iterations; the environment variable GPTQ_IL_MAX_ITERS, read at each call, changes
 * the cap). If the cap is reached first the call still completes with the last iterate and
 * the status word reports GPTQ_ERR_NOT_CONVERGED (info = iterations run). Eigenvalues that
 * are equal at the r-th position make V_r non-unique; they are assumed distinct.
 * H~ = 2 X~^T X~ + lambda~ I with lambda~ = lambda_rel * mean of the n + r diagonal entries
 * of 2 X~^T X~; the first n rows of U~ (H~^-1 = U~^T U~) come from the Schur complement of
 * the extra block, which is positive definite. With r == 0 this is gptq_prepare_hinv +
 * gptq_quantize_layer.
 *   H          device, n x n fp32 raw Hessian 2 X^T X (from gptq_hessian_accumulate).
 *   r          0 <= r <= 128 and r < n.
 *   L          device, n x r fp32 (V_r, columns sorted by decreasing eigenvalue, each
 *              column's largest-magnitude entry positive); unused if r == 0.
 *   R          device, r x m fp32 (row-major); unused if r == 0.
 *   lambda_out device, one fp32: lambda~.
 *   other arguments as in gptq_quantize_layer.
 *   workspace  device, >= gptq_workspace_size(GPTQ_OP_IL_QUANTIZE, m, n, r, block_size).
 * Device errors as in gptq_prepare_hinv and gptq_quantize_layer, and GPTQ_ERR_NOT_CONVERGED.
 */
GPTQ_API int gptq_il_quantize_layer(const void *W, int w_dtype, int64_t m, int64_t n, const float *H,
                           int r, int bits, int group_size, float lambda_rel, int block_size,
                           uint32_t *codes, float *scales, uint8_t *zeros, float *L, float *R,
                           float *lambda_out, double *loss_out, void *workspace,
                           size_t ws_bytes, gptq_stream_t stream);

/*
 * OLrC + Bid-Up refinement of a quantized layer (GPTQ-intrinsic LoRA summary, section 4):
 * `iters` rounds, each first OLrC (the best rank-r L, R for the current codes) and then
 * Bid-Up (one pass of coordinate-wise code updates on the fixed grid for that L, R); the
 * reconstruction error sum_o ||X (w_o - qhat_o - (R^T L^T)_o)||^2 never increases.
 *   OLrC:   E = W - Qhat; P = top-r eigenvectors of E H E^T (m x m, by decreasing
 *           eigenvalue, each column's largest-magnitude entry positive); R = P^T, L = E^T P.
 *   Bid-Up: columns j = 0 .. n-1 in order, all rows at once; the code of (o, j) becomes
 *           clip(rint(c + (d_o H)_j / (H_jj s)), 0, 2^bits - 1) with d_o = w_o - qhat_o -
 *           (R^T L^T)_o and s the row's scale for j's group (scales and zero-points fixed);
 *           columns with H_jj <= 0 are left alone.
 *   W          device, m x n row-major, w_dtype GPTQ_BF16 or GPTQ_F32 (the original weights).
 *   H          device, n x n fp32 raw Hessian 2 X^T X (undamped).
 *   r          0 <= r <= 128, r < m, r < n (r == 0: Bid-Up rounds only, L and R unused).
 *   bits, group_size  the grid of the codes (as in gptq_quantize_layer).
 *   iters      >= 1 rounds.
 *   codes      device, m x (n * bits / 32) uint32, packed as gptq_quantize_layer writes
 *              them: read, and overwritten with the refined codes.
 *   scales, zeros  device, the grid the codes refer to (read only).
 *   L, R       device, n x r and r x m fp32: written with the last round's OLrC result.
 *   loss_hist  device, 2 * iters doubles: the reconstruction error (with X^T X = H / 2)
 *              after each round's OLrC and after its Bid-Up, in order.
 *   workspace  device, >= gptq_workspace_size(GPTQ_OP_IL_REFINE, m, n, r, 0) bytes.
 * The eigenvectors come from the same iteration as in gptq_il_quantize_layer (same stopping
 * rule and cap). Argument errors: GPTQ_ERR_ARG, GPTQ_ERR_WORKSPACE (nothing enqueued). Device
 * errors (a non-positive pivot in the eigenvector step's orthonormalisation, an iteration that
 * reached its cap: GPTQ_ERR_NOT_CONVERGED) go to the status word.
 */
GPTQ_API int gptq_il_refine(const void *W, int w_dtype, int64_t m, int64_t n, const float *H,
                            int r, int bits, int group_size, int iters, uint32_t *codes,
                            const float *scales, const uint8_t *zeros, float *L, float *R,
                            double *loss_hist, void *workspace, size_t ws_bytes,
                            gptq_stream_t stream);

/*
 * Low-precision storage of the low-rank factors (GPTQ-intrinsic LoRA summary, "Main
 * results": quantizing L to 4 bits and R to 8 bits is often lossless). Round-to-nearest,
 * no error feedback, onto the same per-group min-max grid the pass uses, each factor stored
 * one neuron per row like the layer's weights:
 *   L^T: r rows of n inputs, groups of group_size_L (0: one group per row), bits_L;
 *   R^T: m rows of r inputs, one group per row, bits_R.
 *   L, R        device, n x r and r x m fp32 (as gptq_il_quantize_layer / gptq_il_refine
 *               write them), read only.
 *   codes_L     device, r x (n * bits_L / 32) uint32; scales_L r x (n / group size) fp32;
 *               zeros_L the same shape, uint8.
 *   codes_R     device, m x (r * bits_R / 32) uint32; scales_R, zeros_R m x 1.
 *   Codes are packed as gptq_quantize_layer packs them; the dequantized value of code c is
 *   s (c - z). Requires 2 <= bits <= 8, n * bits_L and r * bits_R multiples of 32,
 *   1 <= r <= 128.
 * Argument errors: GPTQ_ERR_ARG (nothing enqueued).
 */
GPTQ_API int gptq_quantize_lowrank(const float *L, const float *R, int64_t n, int64_t m, int r,
                                   int bits_L, int group_size_L, int bits_R, uint32_t *codes_L,
                                   float *scales_L, uint8_t *zeros_L, uint32_t *codes_R,
                                   float *scales_R, uint8_t *zeros_R, gptq_stream_t stream);

/*
 * gptq_2d_round — two-sided adaptive rounding (GPTQ-2D: Cubic-Time Two-Sided Adaptive
 * Rounding, sections 1-2).
 *
 * Finds integers Z for the real matrix X that approximately minimise ||A (Z - X) B||_F^2
 * given the Gram matrices G = A^T A (m x m) and H = B B^T (n x n): the one-sided adaptive
 * rounding of vec X (columns stacked) under H (x) G, run as the anti-diagonal wavefront.
 * Entries are decided in the order of the vectorised sweep up to independence (section 3,
 * Theorems 1 and 2), each as rint(v) with ties to even, v the entry minus the feedback of
 * all earlier errors; there is no grid and no clipping. The feedback factors are the upper
 * U_G, U_H with G^-1 = U_G^T U_G, H^-1 = U_H^T U_H (no damping: A and B are non-singular).
 *
 *   X          device fp32, m x n row-major.
 *   m, n       0 <= m, n <= 65536; m == 0 or n == 0 is a no-op returning GPTQ_OK.
 *   G          device fp32, m x m row-major, symmetric positive definite (upper triangle read).
 *   H          device fp32, n x n row-major, symmetric positive definite (upper triangle read).
 *   Z          device int32, m x n row-major, written. Values outside the int32 range
 *              saturate in Z; the sweep itself continues with the unsaturated integer.
 *   err        device fp32, m x n row-major, written with the errors e = (v - z) / (U_G[p,p]
 *              U_H[q,q]) of the sweep; may be NULL.
 *   workspace  device, >= gptq_workspace_size(GPTQ_OP_2D_ROUND, m, n, 0, 0) bytes, 256-byte
 *              aligned.
 * Returns GPTQ_ERR_ARG (bad pointer or size) or GPTQ_ERR_WORKSPACE before enqueueing
 * anything. Device-side: GPTQ_ERR_NOT_PD if G or H is not numerically positive definite,
 * GPTQ_ERR_NONFINITE (info: the tile row of the entry) if a pre-rounding value is not finite.
 */
GPTQ_API int gptq_2d_round(const float *X, int64_t m, int64_t n, const float *G, const float *H,
                           int32_t *Z, float *err, void *workspace, size_t ws_bytes,
                           gptq_stream_t stream);

/*
 * gptq_quantize_layer_reduced — GPTQ with lattice basis reduction (WITHREDUCTION).
 * The Lattice Geometry of Neural Network Quantization, section 5.2: reduce the basis of the
 * regularised data lattice X' = [X; mu I] (mu^2 = lambda / 2) with LLL before running GPTQ /
 * Babai on it, and map the integer coefficients back through the unimodular change of basis
 * T. The page gives no procedure for the quantization grid; here it is per channel (one min-max
 * scale and zero-point per output row, from the original row: every row's lattice is then s X',
 * so one reduction serves the layer). Steps:
 *   lambda = lambda_rel * mean(diag H); G' = (H + lambda I) / 2 (H's upper triangle read);
 *   LLL (delta = 3/4, fp64, on the Gram matrix) of the column-reversed basis, reversed back:
 *     GPTQ's natural column order is Babai's nearest plane on the reversed basis;
 *   per row: s, z by the min-max rule; u = w / s + z; c' = one-sided adaptive rounding of
 *     T^-1 u under G_red = T^T G' T (rint, ties to even, no clipping);
 *   c = clip(T c', 0, maxq); codes packed as gptq_quantize_layer packs them.
 *   W          device, m x n, w_dtype GPTQ_BF16 or GPTQ_F32; 1 <= m <= 65536.
 *   H          device, n x n fp32 raw Hessian 2 X^T X; 1 <= n <= 2048.
 *   bits       2..8 with n * bits % 32 == 0.
 *   codes      device, m x (n * bits / 32) uint32.  scales, zeros: device, m fp32 / m uint8.
 *   loss_out   device, m fp64 or NULL: (w - w_hat)^T (H + lambda I) (w - w_hat) per row.
 *   coef_out   device, m x n int32 or NULL: the coefficients c' in the reduced basis.
 *   stats_out  device, 8 int64 or NULL: [0] LLL swaps, [1] size reductions, [2] LLL loop
 *              iterations, [3] largest |entry| of T and T^-1, [4] codes that clipping changed,
 *              [5..7] zero.
 *   workspace  device, >= gptq_workspace_size(GPTQ_OP_REDUCED, m, n, 0, 0) bytes.
 * Argument errors: GPTQ_ERR_ARG, GPTQ_ERR_WORKSPACE (nothing enqueued). Device errors:
 * GPTQ_ERR_NOT_PD (G' not numerically positive definite), GPTQ_ERR_NONFINITE (a weight),
 * GPTQ_ERR_NOT_CONVERGED (the LLL loop passed its bound of 64 n^2 + 4096 iterations, info = swaps;
 * or an entry of T beyond 2^24, info = -1).
 */
GPTQ_API int gptq_quantize_layer_reduced(const void *W, int w_dtype, int64_t m, int64_t n,
                                         const float *H, int bits, float lambda_rel,
                                         uint32_t *codes, float *scales, uint8_t *zeros,
                                         double *loss_out, int32_t *coef_out, int64_t *stats_out,
                                         void *workspace, size_t ws_bytes, gptq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_H */
