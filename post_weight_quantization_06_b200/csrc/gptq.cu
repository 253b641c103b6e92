// libgptq: C ABI of the GPTQ / GPTQ-intrinsic-LoRA layer pass for sm_100a.
// One translation unit: the kernels live in the included .cuh files.
#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm_simt.cuh"
#include "factor.cuh"
#include "quant.cuh"
#include "il.cuh"
#include "refine.cuh"
#include "gptq2d.cuh"
#include "hessian_tc.cuh"
#include "lll.cuh"

namespace gptq {

inline size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Carves typed sub-buffers out of the caller's workspace; with base == nullptr it only
// counts, which is how gptq_workspace_size() and the call agree on the layout.
struct Carver {
    char *base;
    size_t off = 0;
    explicit Carver(void *b) : base(static_cast<char *>(b)) {}
    template <typename T>
    T *take(size_t count) {
        T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
        off += align256(count * sizeof(T));
        return p;
    }
};

struct FactorWs {
    float *A, *T;
};
inline FactorWs carve_factor(Carver &c, long long n) {
    FactorWs w;
    w.A = c.take<float>((size_t)n * n);
    w.T = c.take<float>((size_t)FACTOR_T_BLOCKS * FACTOR_NB * n);
    return w;
}

struct QuantWs {
    float *Wc, *Err, *Err_lo, *Uh, *Ul;
};
// Err holds the errors of one outer block of the two-level lazy update: m x OB with
// OB <= min(QUANT_OUTER_MAX, n). With `band`, Uh / Ul hold one outer block's rows of U split
// into tf32 pairs (OB x N each), so that the lazy updates convert nothing; without it (the
// no-allocation entry point's fixed scratch) they are null and the updates split U as they go.
inline QuantWs carve_quant(Carver &c, long long m, long long N, int B, bool band = true) {
    QuantWs w;
    w.Wc = c.take<float>((size_t)m * N);
    const long long ob0 = N < QUANT_OUTER_MAX ? N : QUANT_OUTER_MAX;
    const long long ob = ob0 > B ? ob0 : B;
    w.Err = c.take<float>((size_t)m * ob);
    w.Err_lo = c.take<float>((size_t)m * ob);
    w.Uh = band ? c.take<float>((size_t)ob * N) : nullptr;
    w.Ul = band ? c.take<float>((size_t)ob * N) : nullptr;
    return w;
}

struct IlWs {
    QuantWs q;
    FactorWs f;
    float *Uaug, *lam_dummy;
    ILWork il;
};
// Work arrays of the top-r eigenvector step on a dim x dim matrix.
inline ILWork carve_ilwork(Carver &c, long long dim, int r) {
    ILWork w;
    const int p = il_block_p((int)dim, r);
    w.Y = c.take<float>((size_t)dim * p);
    w.Z = c.take<float>((size_t)dim * p);
    w.HY = c.take<double>((size_t)dim * p);
    w.Tm = c.take<double>((size_t)p * p);
    w.ev = c.take<double>((size_t)p);
    w.Qr = c.take<double>((size_t)p * r);
    w.G = c.take<double>((size_t)p * p);
    w.Gi = c.take<double>((size_t)p * p);
    w.V64 = c.take<double>((size_t)dim * r);
    w.B12 = c.take<double>((size_t)dim * r);
    w.Y1 = c.take<double>((size_t)dim * r);
    w.Yr = c.take<float>((size_t)dim * r);
    w.C = c.take<double>((size_t)r * r);
    w.Ci = c.take<double>((size_t)r * r);
    w.res = c.take<double>((size_t)r * ceil_div(dim, RES_ROWS) + 1);
    w.ctl = c.take<int>(IL_CTL_WORDS);
    w.part_elems = (size_t)4 * dim * p;
    w.part = c.take<double>(w.part_elems);
    return w;
}

inline RefineWs carve_refine(Carver &c, long long m, long long n, int r) {
    RefineWs w;
    w.E = c.take<float>((size_t)m * n);
    w.Gm = c.take<float>((size_t)m * n);
    w.D = c.take<float>((size_t)m * n);
    w.Bm = c.take<float>((size_t)m * m);
    w.P = c.take<float>((size_t)m * (r > 0 ? r : 1));
    w.Z = c.take<float>((size_t)(r > 0 ? r : 1) * n);
    w.Err = c.take<float>((size_t)m * BIDUP_B);
    w.c8 = c.take<uint8_t>((size_t)m * n);
    w.rowloss = c.take<double>((size_t)m);
    if (r > 0) w.il = carve_ilwork(c, m, r);
    else std::memset(&w.il, 0, sizeof(w.il));
    return w;
}

struct TwoDWs {
    FactorWs fg, fh;
    float *UG, *UH, *Xw, *Cacc, *E, *F, *lam;
    long long Mp, Np;
};
// Factors and tile buffers of gptq_2d_round, on the shapes padded to whole 32 x 32 tiles.
inline TwoDWs carve_2d(Carver &c, long long m, long long n) {
    TwoDWs w;
    w.Mp = (m + T2D - 1) / T2D * T2D;
    w.Np = (n + T2D - 1) / T2D * T2D;
    w.fg = carve_factor(c, m);
    w.fh = carve_factor(c, n);
    w.UG = c.take<float>((size_t)(w.Mp * w.Mp));
    w.UH = c.take<float>((size_t)(w.Np * w.Np));
    w.Xw = c.take<float>((size_t)(w.Mp * w.Np));
    w.Cacc = c.take<float>((size_t)(w.Mp * w.Np));
    w.E = c.take<float>((size_t)(w.Mp * w.Np));
    w.F = c.take<float>((size_t)(w.Mp * w.Np));
    w.lam = c.take<float>(2);
    return w;
}

// Buffers of gptq_quantize_layer_reduced.
struct ReducedWs {
    float *lam, *Gd, *A2, *Gred, *Tf, *Tif, *U, *Up, *Cr, *D, *DH;
    double *A, *Bn, *T, *Ti;
    int32_t *Zi;
    uint8_t *c8;
    long long *stats;
    TwoDWs w2;
};
constexpr int REDUCED_STATS = 8;
inline ReducedWs carve_reduced(Carver &c, long long m, long long n) {
    ReducedWs w;
    w.stats = c.take<long long>(REDUCED_STATS);
    w.lam = c.take<float>(2);
    w.A = c.take<double>((size_t)n * n);
    w.Bn = c.take<double>((size_t)n);
    w.T = c.take<double>((size_t)n * n);
    w.Ti = c.take<double>((size_t)n * n);
    w.Gd = c.take<float>((size_t)n * n);
    w.A2 = c.take<float>((size_t)n * n);
    w.Gred = c.take<float>((size_t)n * n);
    w.Tf = c.take<float>((size_t)n * n);
    w.Tif = c.take<float>((size_t)n * n);
    w.U = c.take<float>((size_t)m * n);
    w.Up = c.take<float>((size_t)m * n);
    w.Cr = c.take<float>((size_t)m * n);
    w.D = c.take<float>((size_t)m * n);
    w.DH = c.take<float>((size_t)m * n);
    w.Zi = c.take<int32_t>((size_t)m * n);
    w.c8 = c.take<uint8_t>((size_t)m * n);
    w.w2 = carve_2d(c, m, n);
    return w;
}

inline IlWs carve_il(Carver &c, long long m, long long n, int r, int B) {
    IlWs w;
    w.q = carve_quant(c, m, n + r, B);
    w.f = carve_factor(c, n);
    w.Uaug = c.take<float>((size_t)n * (n + r));
    w.lam_dummy = c.take<float>(1);
    if (r > 0) {
        w.il = carve_ilwork(c, n, r);
    } else {
        std::memset(&w.il, 0, sizeof(w.il));
    }
    return w;
}

inline int check_ws(void *ws, size_t have, size_t need) {
    if (need == 0) return GPTQ_OK;
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) || have < need) return GPTQ_ERR_WORKSPACE;
    return GPTQ_OK;
}

inline bool valid_quant_args(long long m, long long n, int bits, int gs, int B) {
    if (m < 1 || n < 1 || m > (1LL << 30) || n > 65536) return false;
    if (bits < 2 || bits > 8) return false;
    if (B != 32 && B != 64 && B != 128) return false;
    if (n % B) return false;
    if ((n * bits) % 32) return false;
    if (gs < 0) return false;
    if (gs > 0) {
        if (n % gs) return false;
        if (B % gs && gs % B) return false;
    }
    return true;
}

template <typename TX>
int hessian_simt(float *H, const TX *X, long long k, int n, cudaStream_t s) {
    // H(upper) += 2 X^T X, then mirror; chunks of the token axis keep indices in range
    const long long KCH = 1LL << 20;
    for (long long t0 = 0; t0 < k; t0 += KCH) {
        const int kc = (int)((k - t0) < KCH ? (k - t0) : KCH);
        auto p = gemm_args<TX, TX>(n, n, kc, X + t0 * n, n, 1, X + t0 * n, n, 0, H, n, 2.f, 1.f);
        p.c_upper = 1;
        if (int st = gemm_simt(p, s)) return st;
    }
    return mirror_upper(H, n, n, s);
}

int prepare_hinv_impl(const float *H, int n, float lambda_rel, float *U, long long ldu,
                      float *lambda_out, FactorWs &w, cudaStream_t s, int slot = 0) {
    damp_mean_kernel<<<1, 1024, 0, s>>>(H, n, n, lambda_rel, lambda_out);
    GPTQ_CHECK_LAUNCH();
    copy_damped_kernel<<<1184, 256, 0, s>>>(H, n, w.A, n, n, lambda_out);
    GPTQ_CHECK_LAUNCH();
    if (cudaMemsetAsync(U, 0, sizeof(float) * (size_t)n * ldu, s) != cudaSuccess) return GPTQ_ERR_CUDA;
    return factor_ul_inverse(w.A, n, U, ldu, n, w.T, s, slot);
}

int init_work(const void *W, int w_dtype, long long m, int n, float *Wc, long long ldw, int N,
              cudaStream_t s) {
    if (w_dtype == GPTQ_BF16)
        init_work_kernel<__nv_bfloat16><<<1184, 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(W), m, n, Wc, ldw, N);
    else
        init_work_kernel<float><<<1184, 256, 0, s>>>(static_cast<const float *>(W), m, n, Wc, ldw, N);
    return launch_status();
}

// ---------------------------------------------------------------------------------------
// Scratch for gptq_quantize_layer_noalloc: a fixed file-scope device array, so that the
// entry point needs neither a workspace from the caller nor any allocation. Every device
// that loads the library holds it until the process exits. In host code the symbol is only a
// stand-in; its device address is looked up once per device (noalloc_scratch()).
// ---------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[GPTQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
static void *g_noalloc_ptr[kMaxDevices];
static unsigned long long g_noalloc_ctx[kMaxDevices];
static std::mutex g_noalloc_mutex;

// Unique id of the calling thread's current context (never reused within the process), or 0
// when there is no current context or the driver does not provide the call.
inline unsigned long long current_context_id() {
    typedef CUresult (*GetCurrentFn)(CUcontext *);
    typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
    static GetCurrentFn get_current = nullptr;
    static GetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_noalloc_scratch on the current device, or nullptr if the lookup fails.
// The address belongs to the module loaded in one context: it is looked up on the first call
// per device and again whenever that device's current context is not the one it was looked
// up in (e.g. after cudaDeviceReset made the runtime create a new primary context).
inline void *noalloc_scratch() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    const unsigned long long ctx = current_context_id();
    if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
        g_noalloc_ctx[dev] = current_context_id();   // the lookup made the context current
    }
    return g_noalloc_ptr[dev];
}

}  // namespace gptq

using namespace gptq;

extern "C" {

GPTQ_API size_t gptq_workspace_size(int op, int64_t m, int64_t n, int r, int block_size) {
    if (n < 1) return 0;
    Carver c(nullptr);
    switch (op) {
        case GPTQ_OP_HESSIAN:
            return 0;
        case GPTQ_OP_PREPARE_HINV:
            carve_factor(c, n);
            return c.off;
        case GPTQ_OP_QUANTIZE:
            if (m < 1) return 0;
            carve_quant(c, m, n, block_size > 0 ? block_size : 128);
            return c.off;
        case GPTQ_OP_IL_QUANTIZE:
            if (m < 1 || r < 0) return 0;
            carve_il(c, m, n, r, block_size > 0 ? block_size : 128);
            return c.off;
        case GPTQ_OP_IL_REFINE:
            if (m < 1 || r < 0) return 0;
            carve_refine(c, m, n, r);
            return c.off;
        case GPTQ_OP_2D_ROUND:
            if (m < 1 || m > 65536 || n > 65536) return 0;
            carve_2d(c, m, n);
            return c.off;
        case GPTQ_OP_REDUCED:
            if (m < 1 || m > 65536 || n > LLL_MAX_N) return 0;
            carve_reduced(c, m, n);
            return c.off;
        default:
            return 0;
    }
}

GPTQ_API const char *gptq_status_string(int status) {
    switch (status) {
        case GPTQ_OK: return "GPTQ_OK";
        case GPTQ_ERR_ARG: return "GPTQ_ERR_ARG: invalid argument";
        case GPTQ_ERR_NOT_PD: return "GPTQ_ERR_NOT_PD: non-positive pivot in the factorization";
        case GPTQ_ERR_NONFINITE: return "GPTQ_ERR_NONFINITE: NaN or Inf in the input";
        case GPTQ_ERR_TIMEOUT: return "GPTQ_ERR_TIMEOUT: a bounded device wait gave up";
        case GPTQ_ERR_CUDA: return "GPTQ_ERR_CUDA: CUDA runtime error";
        case GPTQ_ERR_WORKSPACE: return "GPTQ_ERR_WORKSPACE: workspace missing, misaligned or too small";
        case GPTQ_ERR_NOT_CONVERGED:
            return "GPTQ_ERR_NOT_CONVERGED: the eigenvector iteration reached its cap before its residual test passed";
        default: return "unknown gptq status";
    }
}

GPTQ_API uint64_t gptq_launch_count(void) { return launch_counter().load(); }

GPTQ_API int gptq_sync_status(gptq_stream_t stream, int64_t *info) {
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) return GPTQ_ERR_CUDA;
    DevStatus st;
    if (cudaMemcpyFromSymbol(&st, g_status, sizeof(st)) != cudaSuccess) return GPTQ_ERR_CUDA;
    DevStatus zero = {0, 0, 0};
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return GPTQ_ERR_CUDA;
    if (info) *info = st.info;
    return st.code;
}

GPTQ_API void gptq_set_flags(unsigned flags) { flags_word().store(flags); }
GPTQ_API unsigned gptq_get_flags(void) { return flags_word().load(); }

GPTQ_API int gptq_kernel_times(gptq_kernel_time *out, int n_out) {
    if (n_out < 0 || (n_out > 0 && !out)) return GPTQ_ERR_ARG;
    std::vector<KtRecord> recs;
    {
        std::lock_guard<std::mutex> lk(kt_log().mu);
        recs.swap(kt_log().recs);
    }
    gptq_kernel_time tot[GPTQ_KT_NCLASSES] = {};
    int st = GPTQ_OK;
    for (const KtRecord &r : recs) {
        float ms = 0.f;
        if (st == GPTQ_OK && (cudaEventSynchronize(r.stop) != cudaSuccess ||
                              cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess))
            st = GPTQ_ERR_CUDA;
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
        if (st != GPTQ_OK || r.cls < 0 || r.cls >= GPTQ_KT_NCLASSES) continue;
        tot[r.cls].launches += 1;
        tot[r.cls].ms += ms;
        tot[r.cls].flops += r.flops;
        tot[r.cls].bytes += r.bytes;
    }
    if (st != GPTQ_OK) return st;
    for (int c = 0; c < n_out && c < GPTQ_KT_NCLASSES; ++c) out[c] = tot[c];
    return GPTQ_KT_NCLASSES;
}

// Applied to the status of every compute entry point once its work is enqueued.
static int finish_call(int st, gptq_stream_t stream) {
    const unsigned f = flags_word().load();
    if (st != GPTQ_OK || !(f & (GPTQ_FLAG_SYNC_STATUS | GPTQ_FLAG_DEBUG_CHECKS))) return st;
    if ((f & GPTQ_FLAG_DEBUG_CHECKS) &&
        (cudaDeviceSynchronize() != cudaSuccess || cudaGetLastError() != cudaSuccess))
        return GPTQ_ERR_CUDA;
    return gptq_sync_status(stream, nullptr);
}

static int gptq_hessian_accumulate_body(float *H, const void *X, int x_dtype, int64_t k, int64_t n,
                                     gptq_stream_t stream) {
    if (!H || !X || k < 0 || n < 1 || n > 65536) return GPTQ_ERR_ARG;
    if (x_dtype != GPTQ_BF16 && x_dtype != GPTQ_F32) return GPTQ_ERR_ARG;
    if (k == 0) return GPTQ_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (x_dtype == GPTQ_BF16) {
        const auto *Xb = static_cast<const __nv_bfloat16 *>(X);
        // tensor-core path: TMA needs a 16-byte aligned base and 16-byte row pitch
        if (n % 8 == 0 && (reinterpret_cast<uintptr_t>(X) & 15u) == 0 &&
            std::getenv("GPTQ_FORCE_SIMT_HESSIAN") == nullptr)
        {
            if (int st = tc::hessian_tc(H, Xb, k, (int)n, s)) return st;
            return mirror_upper(H, n, n, s);
        }
        return hessian_simt(H, Xb, k, (int)n, s);
    }
    // fp32 X: the fp32-accurate tensor-core product (tf32 x 3, both operands split as they
    // load) over the upper triangle; gemm_f32 itself falls back to the SIMT kernel for small or
    // unaligned products
    const auto *Xf = static_cast<const float *>(X);
    if (std::getenv("GPTQ_FORCE_SIMT_HESSIAN") != nullptr) return hessian_simt(H, Xf, k, (int)n, s);
    const long long KCH = 1LL << 30;
    for (long long t0 = 0; t0 < k; t0 += KCH) {
        const int kc = (int)((k - t0) < KCH ? (k - t0) : KCH);
        auto p = gemm_args<float, float>((int)n, (int)n, kc, Xf + t0 * n, n, 1, Xf + t0 * n, n, 0, H,
                                         n, 2.f, 1.f);
        p.c_upper = 1;
        if (int st = gemm_f32(p, s)) return st;
    }
    return mirror_upper(H, n, n, s);
}

GPTQ_API int gptq_hessian_accumulate(float *H, const void *X, int x_dtype, int64_t k, int64_t n,
                                     gptq_stream_t stream) {
    return finish_call(gptq_hessian_accumulate_body(H, X, x_dtype, k, n, stream), stream);
}

static int gptq_prepare_hinv_body(const float *H, int64_t n, float lambda_rel, float *U,
                               float *lambda_out, void *workspace, size_t ws_bytes,
                               gptq_stream_t stream) {
    if (!H || !U || !lambda_out || n < 1 || n > 65536) return GPTQ_ERR_ARG;
    if (!(lambda_rel >= 0.f) || !isfinite(lambda_rel)) return GPTQ_ERR_ARG;
    const size_t need = gptq_workspace_size(GPTQ_OP_PREPARE_HINV, 0, n, 0, 0);
    if (int st = check_ws(workspace, ws_bytes, need)) return st;
    Carver c(workspace);
    FactorWs w = carve_factor(c, n);
    return prepare_hinv_impl(H, (int)n, lambda_rel, U, n, lambda_out, w,
                             reinterpret_cast<cudaStream_t>(stream));
}

GPTQ_API int gptq_prepare_hinv(const float *H, int64_t n, float lambda_rel, float *U,
                               float *lambda_out, void *workspace, size_t ws_bytes,
                               gptq_stream_t stream) {
    const int st = gptq_prepare_hinv_body(H, n, lambda_rel, U, lambda_out, workspace, ws_bytes,
        stream);
    return finish_call(st, stream);
}

static int gptq_quantize_layer_body(const void *W, int w_dtype, int64_t m, int64_t n, const float *U,
                                 int bits, int group_size, int block_size, uint32_t *codes,
                                 float *scales, uint8_t *zeros, double *loss_out,
                                 void *workspace, size_t ws_bytes, gptq_stream_t stream) {
    if (!W || !U || !codes || !scales || !zeros) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_ARG;
    if (!valid_quant_args(m, n, bits, group_size, block_size)) return GPTQ_ERR_ARG;
    const size_t need = gptq_workspace_size(GPTQ_OP_QUANTIZE, m, n, 0, block_size);
    if (int st = check_ws(workspace, ws_bytes, need)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c(workspace);
    QuantWs w = carve_quant(c, m, n, block_size);
    if (int st = init_work(W, w_dtype, m, (int)n, w.Wc, n, (int)n, s)) return st;
    return sweep_layer(w.Wc, n, (int)m, (int)n, (int)n, U, n, bits, group_size, block_size,
                       codes, scales, zeros, loss_out, w.Err, w.Err_lo, w.Uh, w.Ul, s);
}

GPTQ_API int gptq_quantize_layer(const void *W, int w_dtype, int64_t m, int64_t n, const float *U,
                                 int bits, int group_size, int block_size, uint32_t *codes,
                                 float *scales, uint8_t *zeros, double *loss_out,
                                 void *workspace, size_t ws_bytes, gptq_stream_t stream) {
    const int st = gptq_quantize_layer_body(W, w_dtype, m, n, U, bits, group_size, block_size,
        codes, scales, zeros, loss_out, workspace, ws_bytes, stream);
    return finish_call(st, stream);
}

static int gptq_quantize_layer_noalloc_body(const void *W, int w_dtype, int64_t m, int64_t n,
                                         const float *U, int bits, int group_size,
                                         int block_size, uint32_t *codes, float *scales,
                                         uint8_t *zeros, double *loss_out,
                                         gptq_stream_t stream) {
    if (!W || !U || !codes || !scales || !zeros) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_ARG;
    if (!valid_quant_args(m, n, bits, group_size, block_size)) return GPTQ_ERR_ARG;
    Carver sz(nullptr);
    carve_quant(sz, m, n, block_size, false);
    if (sz.off > GPTQ_NOALLOC_SCRATCH_BYTES) return GPTQ_ERR_ARG;
    void *scratch = noalloc_scratch();
    if (!scratch) return GPTQ_ERR_CUDA;
    // The working copy and the per-panel errors are fully written before they are read, so
    // nothing left in the shared scratch by an earlier call needs clearing.
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c(scratch);
    QuantWs w = carve_quant(c, m, n, block_size, false);
    if (int st = init_work(W, w_dtype, m, (int)n, w.Wc, n, (int)n, s)) return st;
    return sweep_layer(w.Wc, n, (int)m, (int)n, (int)n, U, n, bits, group_size, block_size,
                       codes, scales, zeros, loss_out, w.Err, w.Err_lo, nullptr, nullptr, s);
}

GPTQ_API int gptq_quantize_layer_noalloc(const void *W, int w_dtype, int64_t m, int64_t n,
                                         const float *U, int bits, int group_size,
                                         int block_size, uint32_t *codes, float *scales,
                                         uint8_t *zeros, double *loss_out,
                                         gptq_stream_t stream) {
    const int st = gptq_quantize_layer_noalloc_body(W, w_dtype, m, n, U, bits, group_size,
        block_size, codes, scales, zeros, loss_out, stream);
    return finish_call(st, stream);
}

static int gptq_il_quantize_layer_body(const void *W, int w_dtype, int64_t m, int64_t n,
                                    const float *H, int r, int bits, int group_size,
                                    float lambda_rel, int block_size, uint32_t *codes,
                                    float *scales, uint8_t *zeros, float *L, float *R,
                                    float *lambda_out, double *loss_out, void *workspace,
                                    size_t ws_bytes, gptq_stream_t stream) {
    if (!W || !H || !codes || !scales || !zeros || !lambda_out) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_ARG;
    if (!valid_quant_args(m, n, bits, group_size, block_size)) return GPTQ_ERR_ARG;
    if (r < 0 || r > IL_MAX_R || r >= n) return GPTQ_ERR_ARG;
    if (r > 0 && (!L || !R)) return GPTQ_ERR_ARG;
    if (!(lambda_rel >= 0.f) || !isfinite(lambda_rel)) return GPTQ_ERR_ARG;
    const size_t need = gptq_workspace_size(GPTQ_OP_IL_QUANTIZE, m, n, r, block_size);
    if (int st = check_ws(workspace, ws_bytes, need)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c(workspace);
    IlWs w = carve_il(c, m, n, r, block_size);
    const long long N = n + r;
    if (r == 0) {
        if (int st = prepare_hinv_impl(H, (int)n, lambda_rel, w.Uaug, n, lambda_out, w.f, s)) return st;
    } else {
        if (int st = il_top_eigvecs(H, n, (int)n, r, L, w.il, s)) return st;
        if (int st = il_factor(H, n, (int)n, r, lambda_rel, w.Uaug, w.f.A, w.f.T, lambda_out,
                               w.il, s))
            return st;
    }
    if (int st = init_work(W, w_dtype, m, (int)n, w.q.Wc, N, (int)N, s)) return st;
    if (int st = sweep_layer(w.q.Wc, N, (int)m, (int)n, (int)N, w.Uaug, N, bits, group_size,
                             block_size, codes, scales, zeros, loss_out, w.q.Err, w.q.Err_lo,
                             w.q.Uh, w.q.Ul, s))
        return st;
    if (r > 0) {
        extract_R_kernel<<<592, 256, 0, s>>>(w.q.Wc, N, (int)m, (int)n, r, R);
        return launch_status();
    }
    return GPTQ_OK;
}

GPTQ_API int gptq_il_quantize_layer(const void *W, int w_dtype, int64_t m, int64_t n,
                                    const float *H, int r, int bits, int group_size,
                                    float lambda_rel, int block_size, uint32_t *codes,
                                    float *scales, uint8_t *zeros, float *L, float *R,
                                    float *lambda_out, double *loss_out, void *workspace,
                                    size_t ws_bytes, gptq_stream_t stream) {
    const int st = gptq_il_quantize_layer_body(W, w_dtype, m, n, H, r, bits, group_size,
        lambda_rel, block_size, codes, scales, zeros, L, R, lambda_out, loss_out, workspace,
        ws_bytes, stream);
    return finish_call(st, stream);
}

static int gptq_il_refine_body(const void *W, int w_dtype, int64_t m, int64_t n, const float *H,
                            int r, int bits, int group_size, int iters, uint32_t *codes,
                            const float *scales, const uint8_t *zeros, float *L, float *R,
                            double *loss_hist, void *workspace, size_t ws_bytes,
                            gptq_stream_t stream) {
    if (!W || !H || !codes || !scales || !zeros || !loss_hist) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_ARG;
    if (!valid_quant_args(m, n, bits, group_size, 128)) return GPTQ_ERR_ARG;
    if (r < 0 || r > IL_MAX_R || r >= n || r >= m) return GPTQ_ERR_ARG;
    if (r > 0 && (!L || !R)) return GPTQ_ERR_ARG;
    if (iters < 1) return GPTQ_ERR_ARG;
    const size_t need = gptq_workspace_size(GPTQ_OP_IL_REFINE, m, n, r, 0);
    if (int st = check_ws(workspace, ws_bytes, need)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c(workspace);
    RefineWs w = carve_refine(c, m, n, r);
    const int gs = group_size > 0 ? group_size : (int)n;
    const long long words = n * bits / 32;
    const int blocks = (int)std::min<long long>((m * n + 255) / 256, 148LL * 8);
    refine_unpack_kernel<<<blocks, 256, 0, s>>>(codes, words, (int)m, (int)n, bits, w.c8, n);
    GPTQ_CHECK_LAUNCH();
    int st;
    if (w_dtype == GPTQ_BF16)
        st = il_refine(static_cast<const __nv_bfloat16 *>(W), (int)m, (int)n, H, r, bits, gs,
                       iters, scales, zeros, L, R, loss_hist, w, s);
    else
        st = il_refine(static_cast<const float *>(W), (int)m, (int)n, H, r, bits, gs, iters,
                       scales, zeros, L, R, loss_hist, w, s);
    if (st) return st;
    refine_pack_kernel<<<blocks, 256, 0, s>>>(w.c8, n, (int)m, (int)n, bits, codes, words);
    return launch_status();
}

GPTQ_API int gptq_il_refine(const void *W, int w_dtype, int64_t m, int64_t n, const float *H,
                            int r, int bits, int group_size, int iters, uint32_t *codes,
                            const float *scales, const uint8_t *zeros, float *L, float *R,
                            double *loss_hist, void *workspace, size_t ws_bytes,
                            gptq_stream_t stream) {
    const int st = gptq_il_refine_body(W, w_dtype, m, n, H, r, bits, group_size, iters, codes,
        scales, zeros, L, R, loss_hist, workspace, ws_bytes, stream);
    return finish_call(st, stream);
}

static int gptq_quantize_lowrank_body(const float *L, const float *R, int64_t n, int64_t m, int r,
                                   int bits_L, int group_size_L, int bits_R, uint32_t *codes_L,
                                   float *scales_L, uint8_t *zeros_L, uint32_t *codes_R,
                                   float *scales_R, uint8_t *zeros_R, gptq_stream_t stream) {
    if (!L || !R || !codes_L || !scales_L || !zeros_L || !codes_R || !scales_R || !zeros_R)
        return GPTQ_ERR_ARG;
    if (n < 1 || m < 1 || r < 1 || r > IL_MAX_R || n > 65536 || m > (1LL << 30)) return GPTQ_ERR_ARG;
    if (bits_L < 2 || bits_L > 8 || bits_R < 2 || bits_R > 8) return GPTQ_ERR_ARG;
    if ((n * bits_L) % 32 || ((long long)r * bits_R) % 32) return GPTQ_ERR_ARG;
    if (group_size_L < 0 || (group_size_L > 0 && n % group_size_L)) return GPTQ_ERR_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int gsL = group_size_L > 0 ? group_size_L : (int)n;
    // L^T: r rows of n inputs; R^T: m rows of r inputs (one group)
    rtn_rows_kernel<<<ceil_div(r, 8), 256, 0, s>>>(L, 1, r, r, (int)n, bits_L, gsL, codes_L,
                                                   n * bits_L / 32, scales_L, zeros_L,
                                                   (int)(n / gsL));
    GPTQ_CHECK_LAUNCH();
    rtn_rows_kernel<<<ceil_div(m, 8), 256, 0, s>>>(R, 1, m, (int)m, r, bits_R, r, codes_R,
                                                   (long long)r * bits_R / 32, scales_R, zeros_R, 1);
    return launch_status();
}

GPTQ_API int gptq_quantize_lowrank(const float *L, const float *R, int64_t n, int64_t m, int r,
                                   int bits_L, int group_size_L, int bits_R, uint32_t *codes_L,
                                   float *scales_L, uint8_t *zeros_L, uint32_t *codes_R,
                                   float *scales_R, uint8_t *zeros_R, gptq_stream_t stream) {
    const int st = gptq_quantize_lowrank_body(L, R, n, m, r, bits_L, group_size_L, bits_R,
        codes_L, scales_L, zeros_L, codes_R, scales_R, zeros_R, stream);
    return finish_call(st, stream);
}

static int gptq_2d_round_body(const float *X, int64_t m, int64_t n, const float *G, const float *H,
                           int32_t *Z, float *err, void *workspace, size_t ws_bytes,
                           gptq_stream_t stream) {
    if (m < 0 || n < 0 || m > 65536 || n > 65536) return GPTQ_ERR_ARG;
    if (m == 0 || n == 0) return GPTQ_OK;
    if (!X || !G || !H || !Z) return GPTQ_ERR_ARG;
    const size_t need = gptq_workspace_size(GPTQ_OP_2D_ROUND, m, n, 0, 0);
    if (int st = check_ws(workspace, ws_bytes, need)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c(workspace);
    TwoDWs w = carve_2d(c, m, n);
    // U_G (side stream, second factor slot) and U_H (this stream) at once, no damping;
    // identity rows on the padding
    Gptq2dSide *side = gptq2d_side();
    if (!side) return GPTQ_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(side->mu);
        if (cudaEventRecord(side->fork, s) != cudaSuccess ||
            cudaStreamWaitEvent(side->stream, side->fork, 0) != cudaSuccess)
            return GPTQ_ERR_CUDA;
        if (int st = prepare_hinv_impl(G, (int)m, 0.f, w.UG, w.Mp, w.lam + 1, w.fg, side->stream, 1))
            return st;
        if (w.Mp > m) {
            gptq2d_pad_identity_kernel<<<64, 256, 0, side->stream>>>(w.UG, m, w.Mp);
            GPTQ_CHECK_LAUNCH();
        }
        if (cudaEventRecord(side->join, side->stream) != cudaSuccess) return GPTQ_ERR_CUDA;
        if (int st = prepare_hinv_impl(H, (int)n, 0.f, w.UH, w.Np, w.lam, w.fh, s, 0)) return st;
        if (w.Np > n) {
            gptq2d_pad_identity_kernel<<<64, 256, 0, s>>>(w.UH, n, w.Np);
            GPTQ_CHECK_LAUNCH();
        }
        if (cudaStreamWaitEvent(s, side->join, 0) != cudaSuccess) return GPTQ_ERR_CUDA;
    }
    gptq2d_init_kernel<<<1184, 256, 0, s>>>(X, (int)m, (int)n, w.Xw, w.Cacc, w.Mp, w.Np);
    GPTQ_CHECK_LAUNCH();
    Gptq2dArgs a;
    a.Xw = w.Xw; a.Cacc = w.Cacc; a.E = w.E; a.F = w.F; a.UG = w.UG; a.UH = w.UH;
    a.Z = Z; a.err = err; a.Mp = w.Mp; a.Np = w.Np; a.m = (int)m; a.n = (int)n;
    a.MT = (int)(w.Mp / T2D); a.NT = (int)(w.Np / T2D);
    return gptq2d_sweep(a, s);
}

GPTQ_API int gptq_2d_round(const float *X, int64_t m, int64_t n, const float *G, const float *H,
                           int32_t *Z, float *err, void *workspace, size_t ws_bytes,
                           gptq_stream_t stream) {
    const int st = gptq_2d_round_body(X, m, n, G, H, Z, err, workspace, ws_bytes, stream);
    return finish_call(st, stream);
}

static int gptq_quantize_layer_reduced_body(const void *W, int w_dtype, int64_t m, int64_t n,
                                            const float *H, int bits, float lambda_rel,
                                            uint32_t *codes, float *scales, uint8_t *zeros,
                                            double *loss_out, int32_t *coef_out,
                                            int64_t *stats_out, void *workspace, size_t ws_bytes,
                                            gptq_stream_t stream) {
    if (!W || !H || !codes || !scales || !zeros) return GPTQ_ERR_ARG;
    if (w_dtype != GPTQ_BF16 && w_dtype != GPTQ_F32) return GPTQ_ERR_ARG;
    if (m < 1 || m > 65536 || n < 1 || n > LLL_MAX_N) return GPTQ_ERR_ARG;
    if (bits < 2 || bits > 8 || (n * bits) % 32) return GPTQ_ERR_ARG;
    if (!(lambda_rel >= 0.f) || !isfinite(lambda_rel)) return GPTQ_ERR_ARG;
    const size_t need = gptq_workspace_size(GPTQ_OP_REDUCED, m, n, 0, 0);
    if (int st = check_ws(workspace, ws_bytes, need)) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Carver c(workspace);
    ReducedWs w = carve_reduced(c, m, n);
    const int N = (int)n, M = (int)m;
    const long long mn = m * n;
    const int blocks = (int)std::min<long long>((std::max<long long>(mn, n * n) + 255) / 256, 148LL * 8);
    if (cudaMemsetAsync(w.stats, 0, sizeof(long long) * REDUCED_STATS, s) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    // lambda, G' = (H + lambda I) / 2, its LLL reduction T (and T^-1) for GPTQ's column order
    damp_mean_kernel<<<1, 1024, 0, s>>>(H, n, N, lambda_rel, w.lam);
    GPTQ_CHECK_LAUNCH();
    lll_prep_kernel<<<blocks, 256, 0, s>>>(H, n, N, w.lam, w.A, w.Gd);
    GPTQ_CHECK_LAUNCH();
    lll_kernel<<<1, LLL_THREADS, 0, s>>>(w.A, N, w.Bn, w.T, w.Ti, w.stats, 64LL * n * n + 4096,
                                         0.75);
    GPTQ_CHECK_LAUNCH();
    lll_export_kernel<<<blocks, 256, 0, s>>>(w.T, w.Ti, N, w.Tf, w.Tif, w.stats);
    GPTQ_CHECK_LAUNCH();
    // G_red = T^T G' T
    if (int st = gemm_f32(gemm_args<float, float>(N, N, N, w.Gd, n, 0, w.Tf, n, 0, w.A2, n, 1.f,
                                                  0.f), s)) return st;
    if (int st = gemm_f32(gemm_args<float, float>(N, N, N, w.Tf, n, 1, w.A2, n, 0, w.Gred, n, 1.f,
                                                  0.f), s)) return st;
    // per-channel grid and the grid coordinates in the reduced basis, u' = T^-1 u
    if (w_dtype == GPTQ_BF16)
        rowgrid_kernel<__nv_bfloat16><<<ceil_div(m, 8), 256, 0, s>>>(
            static_cast<const __nv_bfloat16 *>(W), M, N, bits, scales, zeros, w.U);
    else
        rowgrid_kernel<float><<<ceil_div(m, 8), 256, 0, s>>>(static_cast<const float *>(W), M, N,
                                                              bits, scales, zeros, w.U);
    GPTQ_CHECK_LAUNCH();
    if (int st = gemm_f32(gemm_args<float, float>(M, N, N, w.U, n, 0, w.Tif, n, 1, w.Up, n, 1.f,
                                                  0.f), s)) return st;
    // Babai in the reduced basis: one-sided adaptive rounding of u' under G_red (the two-sided
    // wavefront with U_G = I)
    TwoDWs &t = w.w2;
    gptq2d_pad_identity_kernel<<<64, 256, 0, s>>>(t.UG, 0, t.Mp);
    GPTQ_CHECK_LAUNCH();
    if (int st = prepare_hinv_impl(w.Gred, N, 0.f, t.UH, t.Np, t.lam, t.fh, s, 0)) return st;
    if (t.Np > n) {
        gptq2d_pad_identity_kernel<<<64, 256, 0, s>>>(t.UH, n, t.Np);
        GPTQ_CHECK_LAUNCH();
    }
    gptq2d_init_kernel<<<1184, 256, 0, s>>>(w.Up, M, N, t.Xw, t.Cacc, t.Mp, t.Np);
    GPTQ_CHECK_LAUNCH();
    Gptq2dArgs a;
    a.Xw = t.Xw; a.Cacc = t.Cacc; a.E = t.E; a.F = t.F; a.UG = t.UG; a.UH = t.UH;
    a.Z = w.Zi; a.err = nullptr; a.Mp = t.Mp; a.Np = t.Np; a.m = M; a.n = N;
    a.MT = (int)(t.Mp / T2D); a.NT = (int)(t.Np / T2D);
    if (int st = gptq2d_sweep(a, s)) return st;
    if (coef_out &&
        cudaMemcpyAsync(coef_out, w.Zi, sizeof(int32_t) * mn, cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
        return GPTQ_ERR_CUDA;
    // back to the original coordinates: c = clip(T c'), codes, loss
    int_to_float_kernel<<<blocks, 256, 0, s>>>(w.Zi, mn, w.U);
    GPTQ_CHECK_LAUNCH();
    if (int st = gemm_f32(gemm_args<float, float>(M, N, N, w.U, n, 0, w.Tf, n, 1, w.Cr, n, 1.f,
                                                  0.f), s)) return st;
    if (w_dtype == GPTQ_BF16)
        reduced_codes_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
            w.Cr, static_cast<const __nv_bfloat16 *>(W), scales, zeros, M, N, bits, w.c8, w.D,
            w.stats);
    else
        reduced_codes_kernel<float><<<blocks, 256, 0, s>>>(w.Cr, static_cast<const float *>(W),
                                                           scales, zeros, M, N, bits, w.c8, w.D,
                                                           w.stats);
    GPTQ_CHECK_LAUNCH();
    pack_codes_kernel<<<blocks, 256, 0, s>>>(w.c8, M, N, bits, codes);
    GPTQ_CHECK_LAUNCH();
    if (loss_out) {
        // (w - w_hat)^T (H + lambda I) (w - w_hat) = 2 d G' d^T
        if (int st = gemm_f32(gemm_args<float, float>(M, N, N, w.D, n, 0, w.Gd, n, 0, w.DH, n,
                                                      2.f, 0.f), s)) return st;
        refine_rowdot_kernel<<<ceil_div(m, 8), 256, 0, s>>>(w.D, w.DH, M, N, loss_out);
        GPTQ_CHECK_LAUNCH();
    }
    if (stats_out &&
        cudaMemcpyAsync(stats_out, w.stats, sizeof(long long) * REDUCED_STATS,
                        cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return GPTQ_ERR_CUDA;
    return GPTQ_OK;
}

GPTQ_API int gptq_quantize_layer_reduced(const void *W, int w_dtype, int64_t m, int64_t n,
                                         const float *H, int bits, float lambda_rel,
                                         uint32_t *codes, float *scales, uint8_t *zeros,
                                         double *loss_out, int32_t *coef_out, int64_t *stats_out,
                                         void *workspace, size_t ws_bytes, gptq_stream_t stream) {
    const int st = gptq_quantize_layer_reduced_body(W, w_dtype, m, n, H, bits, lambda_rel, codes,
        scales, zeros, loss_out, coef_out, stats_out, workspace, ws_bytes, stream);
    return finish_call(st, stream);
}

}  // extern "C"
