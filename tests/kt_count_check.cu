// Host-only check of the GEMM work counts behind gptq_kernel_times: the closed-form flops and
// bytes of kt_count against a brute-force count over every (i, j, k) of random small shapes
// with every combination of the triangular structure flags. Prints the number of mismatches;
// exit status 0 when there are none.
#include <cstdio>
#include <random>

#include "gemm_simt.cuh"

int main() {
    using namespace gptq;
    std::mt19937 rng(12345);
    int bad = 0, cases = 0;
    for (int t = 0; t < 3000; ++t) {
        const int M = 1 + rng() % 37, N = 1 + rng() % 37, K = 1 + rng() % 37;
        GemmArgs<float, float> g = gemm_args<float, float>(M, N, K, nullptr, 0, 0, nullptr, 0, 0,
                                                           nullptr, 0, 1.f, (rng() & 1) ? 1.f : 0.f);
        g.c_upper = rng() & 1;
        g.a_upper = rng() & 1;
        g.a_lower = rng() & 1;
        g.b_upper = rng() & 1;
        g.b_lower = rng() & 1;
        double flops, bytes;
        kt_count(g, flops, bytes);
        double bf = 0, a_nz = 0, b_nz = 0, c_w = 0;
        for (int i = 0; i < M; ++i)
            for (int j = 0; j < N; ++j) {
                if (g.c_upper && j < i) continue;
                c_w += 1;
                for (int k = 0; k < K; ++k) {
                    const bool a = !(g.a_upper && k < i) && !(g.a_lower && k > i);
                    const bool b = !(g.b_upper && k > j) && !(g.b_lower && k < j);
                    if (a && b) bf += 2;
                }
            }
        for (int i = 0; i < M; ++i)
            for (int k = 0; k < K; ++k) a_nz += !(g.a_upper && k < i) && !(g.a_lower && k > i);
        for (int j = 0; j < N; ++j)
            for (int k = 0; k < K; ++k) b_nz += !(g.b_upper && k > j) && !(g.b_lower && k < j);
        const double bb = 4 * (a_nz + b_nz) + 4 * c_w * (g.beta != 0.f ? 2 : 1);
        ++cases;
        if (bf != flops || bb != bytes) {
            if (bad < 5)
                std::printf("M %d N %d K %d c_upper %d a_upper %d a_lower %d b_upper %d b_lower %d: "
                            "flops %.0f vs %.0f, bytes %.0f vs %.0f\n",
                            M, N, K, g.c_upper, g.a_upper, g.a_lower, g.b_upper, g.b_lower, flops,
                            bf, bytes, bb);
            ++bad;
        }
    }
    std::printf("%d of %d cases differ\n", bad, cases);
    return bad != 0;
}
