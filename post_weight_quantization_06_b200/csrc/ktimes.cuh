// Opt-in device timing of the library's fp32 GEMM launches (GPTQ_FLAG_KERNEL_TIMES).
//
// While the flag is set, every launch of the fp32 GEMM (the tf32 x 3 tensor-core kernel and the
// SIMT kernel) is bracketed by two CUDA events on its stream and tagged with the stage that
// issued it (factor, column sweep, intrinsic LoRA, refinement, two-sided rounding) and with its
// algorithmic flops and bytes; gptq_kernel_times() waits for the events and sums them per
// class. Host code only; with the flag clear nothing is recorded and no event is created.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"

namespace gptq {

template <typename TA, typename TB> struct GemmArgs;

// Process-wide behaviour flags (gptq_set_flags).
inline std::atomic<unsigned> &flags_word() {
    static std::atomic<unsigned> f{0};
    return f;
}

// Stages are gptq_kt_stage (gptq.h); class index = stage * 2 + path.
enum KtPath { KT_TC = 0, KT_SIMT = 1 };
static_assert(GPTQ_KT_NCLASSES == 2 * GPTQ_KT_NSTAGES, "one class per stage and path");

inline int &kt_stage() {
    static thread_local int s = GPTQ_KT_OTHER;
    return s;
}

// Attributes the GEMM launches issued inside its lifetime to one stage (nests).
struct KtStageScope {
    int prev;
    explicit KtStageScope(int s) : prev(kt_stage()) { kt_stage() = s; }
    ~KtStageScope() { kt_stage() = prev; }
    KtStageScope(const KtStageScope &) = delete;
    KtStageScope &operator=(const KtStageScope &) = delete;
};

struct KtRecord {
    cudaEvent_t start, stop;
    int cls;
    double flops, bytes;
};

struct KtLog {
    std::mutex mu;
    std::vector<KtRecord> recs;
};

inline KtLog &kt_log() {
    static KtLog l;
    return l;
}

inline bool kt_enabled() {
    return (flags_word().load(std::memory_order_relaxed) & GPTQ_FLAG_KERNEL_TIMES) != 0;
}

// sum over integer j in [j0, j1) of max(0, min(H, bu ? j + 1 : H) - max(L, bl ? j : L)):
// the number of k in [L, H) with (bu: k <= j) and (bl: k >= j), summed over the columns j of
// one output row. The summand is piecewise linear in j with kinks and zero crossings only at
// L - 1, L, H - 1, H, so it is summed exactly segment by segment.
inline double kt_row_products(long long L, long long H, long long j0, long long j1, bool bu,
                              bool bl) {
    if (j1 <= j0 || H <= L) return 0.0;
    auto f = [&](long long j) -> double {
        const long long hi = bu ? std::min(H, j + 1) : H;
        const long long lo = bl ? std::max(L, j) : L;
        return hi > lo ? (double)(hi - lo) : 0.0;
    };
    long long cut[6] = {j0, L - 1, L, H - 1, H, j1};
    std::sort(cut, cut + 6);
    double total = 0.0;
    for (int c = 0; c < 5; ++c) {
        const long long p = std::max(cut[c], j0), q = std::min(cut[c + 1], j1);
        if (q <= p) continue;
        total += (double)(q - p) * (f(p) + f(q - 1)) * 0.5;
    }
    return total;
}

// Algorithmic work of C = alpha op(A) op(B) + beta C with the GemmArgs structure flags:
// flops = 2 x the multiply-adds whose factors are both structurally nonzero, over the entries
// of C that are written; bytes = every structurally nonzero operand element read once, every
// written entry of C stored once (and loaded once when beta != 0).
template <typename TA, typename TB>
inline void kt_count(const GemmArgs<TA, TB> &g, double &flops, double &bytes) {
    flops = 0.0;
    double a_elems = 0.0, b_elems = 0.0, c_elems = 0.0;
    const long long K = g.K, N = g.N;
    for (long long i = 0; i < g.M; ++i) {
        const long long L = g.a_upper ? std::min(i, K) : 0;
        const long long H = g.a_lower ? std::min(i + 1, K) : K;
        const long long j0 = g.c_upper ? i : 0;
        flops += 2.0 * kt_row_products(L, H, j0, N, g.b_upper != 0, g.b_lower != 0);
        a_elems += (double)std::max(0LL, H - L);
        c_elems += (double)std::max(0LL, N - j0);
    }
    for (long long j = 0; j < N; ++j) {
        const long long L = g.b_lower ? std::min(j, K) : 0;
        const long long H = g.b_upper ? std::min(j + 1, K) : K;
        b_elems += (double)std::max(0LL, H - L);
    }
    bytes = a_elems * sizeof(TA) + b_elems * sizeof(TB) +
            c_elems * sizeof(float) * (g.beta != 0.f ? 2.0 : 1.0);
}

// Brackets one launch on stream s; inert unless the flag is set, and for a conditional launch
// (one that a device flag may turn into a no-op, whose work is therefore not known here).
struct KtSpan {
    bool on;
    cudaStream_t s;
    cudaEvent_t a = nullptr, b = nullptr;
    explicit KtSpan(cudaStream_t st, bool conditional = false)
        : on(kt_enabled() && !conditional), s(st) {
        if (!on) return;
        if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess ||
            cudaEventRecord(a, s) != cudaSuccess) {
            if (a) cudaEventDestroy(a);
            if (b) cudaEventDestroy(b);
            a = b = nullptr;
            on = false;
        }
    }
    template <typename TA, typename TB>
    void done(int path, const GemmArgs<TA, TB> &g) {
        if (!on) return;
        on = false;
        if (cudaEventRecord(b, s) != cudaSuccess) {
            cudaEventDestroy(a);
            cudaEventDestroy(b);
            return;
        }
        KtRecord r;
        r.start = a;
        r.stop = b;
        r.cls = kt_stage() * 2 + path;
        kt_count(g, r.flops, r.bytes);
        std::lock_guard<std::mutex> lk(kt_log().mu);
        kt_log().recs.push_back(r);
    }
    ~KtSpan() {
        if (on) {  // launch path returned before done(): drop the pair
            cudaEventDestroy(a);
            cudaEventDestroy(b);
        }
    }
    KtSpan(const KtSpan &) = delete;
    KtSpan &operator=(const KtSpan &) = delete;
};

}  // namespace gptq
