// fp64 matrix product and host threading of the C++ oracle.
//
// TEST INFRASTRUCTURE ONLY: this file belongs to the oracle, which only the
// tests, the smoke check and the benchmark's host baseline use.  It shares no
// code with the CUDA library.
//
// The matrix product is the one library-style primitive the oracle's
// Newton-Schulz iteration leans on.  Its definition is the textbook one,
//     C[i][j] = sum_{k = 0 .. K-1} op(A)[i][k] op(B)[k][j],
// with the sum taken in ascending k and every term added by one fused
// multiply-add (acc <- fma(a_ik, b_kj, acc), acc = +0 before the first term).
// The loops below are blocked for the host caches, but blocking only changes
// where the running sum of an element waits between two terms (a register, or
// C itself between K blocks); the terms, their order and every rounding are
// those of the definition, so the result is bit for bit the plain triple loop.
// The pins (tests/test_oracle_native.py) check exactly that against an
// exact-rational replay of the definition, and against numpy's product.
#include "oracle_f64.h"

#include <sched.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

#if defined(__x86_64__)
#include <immintrin.h>
#endif

namespace oracle {

// ---------------------------------------------------------------------------
// threads
// ---------------------------------------------------------------------------
namespace {

int default_threads() {
    if (const char* e = std::getenv("ORACLE_THREADS")) {
        const int v = std::atoi(e);
        if (v > 0) return v;
    }
    cpu_set_t set;
    if (sched_getaffinity(0, sizeof(set), &set) == 0) {
        const int n = CPU_COUNT(&set);
        if (n > 0) return n;
    }
    const unsigned h = std::thread::hardware_concurrency();
    return h > 0 ? static_cast<int>(h) : 1;
}

std::atomic<int> g_threads{0};

}  // namespace

int threads() {
    int t = g_threads.load();
    if (t <= 0) {
        t = default_threads();
        g_threads.store(t);
    }
    return t;
}

void set_threads(int t) { g_threads.store(t > 0 ? t : default_threads()); }

void parallel_for(int64_t ntasks, const std::function<void(int64_t)>& body) {
    if (ntasks <= 0) return;
    const int nt = static_cast<int>(std::min<int64_t>(threads(), ntasks));
    if (nt <= 1) {
        for (int64_t t = 0; t < ntasks; ++t) body(t);
        return;
    }
    std::atomic<int64_t> next{0};
    auto worker = [&] {
        for (int64_t t = next.fetch_add(1); t < ntasks; t = next.fetch_add(1)) body(t);
    };
    std::vector<std::thread> pool;
    pool.reserve(nt - 1);
    for (int i = 0; i < nt - 1; ++i) pool.emplace_back(worker);
    worker();
    for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------------
// matrix product
// ---------------------------------------------------------------------------
namespace {

constexpr int MR = 6;          // rows of C per register tile
constexpr int NR = 16;         // columns of C per register tile
constexpr int64_t MC = 96;     // rows of C per task (a multiple of MR)
constexpr int64_t NC = 512;    // columns of C per task (a multiple of NR)
constexpr int64_t KC = 256;    // terms per K block

struct Operand {
    const double* p;
    int64_t ld;
    bool trans;
};

// op(A) rows [i0, i0 + mc) x terms [k0, k0 + kc), as panels of MR rows:
// panel q holds element (i0 + q MR + r, k0 + k) at q * kc * MR + k * MR + r;
// rows past the block are zero.
void pack_a(const Operand& A, int64_t i0, int64_t mc, int64_t k0, int64_t kc, double* out) {
    for (int64_t q = 0; q * MR < mc; ++q) {
        double* panel = out + q * kc * MR;
        const int live = static_cast<int>(std::min<int64_t>(MR, mc - q * MR));
        const int64_t ib = i0 + q * MR;
        if (A.trans) {            // element (i, k) at A[k * ld + i]: rows of the panel are contiguous
            for (int64_t k = 0; k < kc; ++k)
                for (int r = 0; r < MR; ++r) panel[k * MR + r] = r < live ? A.p[(k0 + k) * A.ld + ib + r] : 0.0;
        } else {                  // element (i, k) at A[i * ld + k]: terms are contiguous
            for (int r = 0; r < MR; ++r)
                for (int64_t k = 0; k < kc; ++k) panel[k * MR + r] = r < live ? A.p[(ib + r) * A.ld + k0 + k] : 0.0;
        }
    }
}

// op(B) terms [k0, k0 + kc) x columns [j0, j0 + nc), as panels of NR columns:
// panel q holds element (k0 + k, j0 + q NR + c) at q * kc * NR + k * NR + c;
// columns past the block are zero.
void pack_b(const Operand& B, int64_t j0, int64_t nc, int64_t k0, int64_t kc, double* out) {
    for (int64_t q = 0; q * NR < nc; ++q) {
        double* panel = out + q * kc * NR;
        const int live = static_cast<int>(std::min<int64_t>(NR, nc - q * NR));
        const int64_t jb = j0 + q * NR;
        if (B.trans) {            // element (k, j) at B[j * ld + k]: terms are contiguous
            for (int c = 0; c < NR; ++c)
                for (int64_t k = 0; k < kc; ++k) panel[k * NR + c] = c < live ? B.p[(jb + c) * B.ld + k0 + k] : 0.0;
        } else {                  // element (k, j) at B[k * ld + j]: columns of the panel are contiguous
            for (int64_t k = 0; k < kc; ++k)
                for (int c = 0; c < NR; ++c) panel[k * NR + c] = c < live ? B.p[(k0 + k) * B.ld + jb + c] : 0.0;
        }
    }
}

// One MR x NR tile: acc[r][c] <- fma(Ap[k][r], Bp[k][c], acc[r][c]) for
// k = 0 .. kc-1 in order, acc starting from C (first == false) or +0.
// Portable form; the vector forms below compute exactly this, one lane per
// element.
void tile_scalar(int64_t kc, const double* Ap, const double* Bp, double* C, int64_t ldc, bool first) {
    double acc[MR][NR];
    for (int r = 0; r < MR; ++r)
        for (int c = 0; c < NR; ++c) acc[r][c] = first ? 0.0 : C[r * ldc + c];
    for (int64_t k = 0; k < kc; ++k)
        for (int r = 0; r < MR; ++r)
            for (int c = 0; c < NR; ++c) acc[r][c] = std::fma(Ap[k * MR + r], Bp[k * NR + c], acc[r][c]);
    for (int r = 0; r < MR; ++r)
        for (int c = 0; c < NR; ++c) C[r * ldc + c] = acc[r][c];
}

#if defined(__x86_64__)
// Accumulators are named variables (not arrays) so that they stay in registers.
#define ORACLE_ROWS(X) X(0) X(1) X(2) X(3) X(4) X(5)

// 8-wide lanes: the 6 x 16 tile as 6 x 2 vectors.
__attribute__((target("avx512f"))) void tile_avx512(int64_t kc, const double* Ap, const double* Bp, double* C,
                                                    int64_t ldc, bool first) {
#define DECL(r) __m512d c##r##0 = first ? _mm512_setzero_pd() : _mm512_loadu_pd(C + r * ldc);       \
                __m512d c##r##1 = first ? _mm512_setzero_pd() : _mm512_loadu_pd(C + r * ldc + 8);
    ORACLE_ROWS(DECL)
#undef DECL
    for (int64_t k = 0; k < kc; ++k) {
        const __m512d b0 = _mm512_loadu_pd(Bp + k * NR);
        const __m512d b1 = _mm512_loadu_pd(Bp + k * NR + 8);
#define STEP(r) { const __m512d a = _mm512_set1_pd(Ap[k * MR + r]);                                  \
                  c##r##0 = _mm512_fmadd_pd(a, b0, c##r##0); c##r##1 = _mm512_fmadd_pd(a, b1, c##r##1); }
        ORACLE_ROWS(STEP)
#undef STEP
    }
#define STORE(r) _mm512_storeu_pd(C + r * ldc, c##r##0); _mm512_storeu_pd(C + r * ldc + 8, c##r##1);
    ORACLE_ROWS(STORE)
#undef STORE
}

// 4-wide lanes: half of the tile's columns (8) per call, as 6 x 2 vectors.
__attribute__((target("avx2,fma"))) void half_tile_avx2(int64_t kc, const double* Ap, const double* Bp, double* C,
                                                        int64_t ldc, bool first) {
#define DECL(r) __m256d c##r##0 = first ? _mm256_setzero_pd() : _mm256_loadu_pd(C + r * ldc);       \
                __m256d c##r##1 = first ? _mm256_setzero_pd() : _mm256_loadu_pd(C + r * ldc + 4);
    ORACLE_ROWS(DECL)
#undef DECL
    for (int64_t k = 0; k < kc; ++k) {
        const __m256d b0 = _mm256_loadu_pd(Bp + k * NR);
        const __m256d b1 = _mm256_loadu_pd(Bp + k * NR + 4);
#define STEP(r) { const __m256d a = _mm256_broadcast_sd(Ap + k * MR + r);                            \
                  c##r##0 = _mm256_fmadd_pd(a, b0, c##r##0); c##r##1 = _mm256_fmadd_pd(a, b1, c##r##1); }
        ORACLE_ROWS(STEP)
#undef STEP
    }
#define STORE(r) _mm256_storeu_pd(C + r * ldc, c##r##0); _mm256_storeu_pd(C + r * ldc + 4, c##r##1);
    ORACLE_ROWS(STORE)
#undef STORE
}
#undef ORACLE_ROWS

enum class Isa { Scalar, Avx2, Avx512 };

Isa isa() {
    static const Isa v = __builtin_cpu_supports("avx512f") ? Isa::Avx512
                         : (__builtin_cpu_supports("avx2") && __builtin_cpu_supports("fma")) ? Isa::Avx2
                                                                                             : Isa::Scalar;
    return v;
}
#endif

void tile(int64_t kc, const double* Ap, const double* Bp, double* C, int64_t ldc, bool first) {
#if defined(__x86_64__)
    switch (isa()) {
        case Isa::Avx512: tile_avx512(kc, Ap, Bp, C, ldc, first); return;
        case Isa::Avx2:
            half_tile_avx2(kc, Ap, Bp, C, ldc, first);
            half_tile_avx2(kc, Ap, Bp + 8, C + 8, ldc, first);
            return;
        default: break;
    }
#endif
    tile_scalar(kc, Ap, Bp, C, ldc, first);
}

}  // namespace

void matmul(int64_t M, int64_t N, int64_t K, const double* A, int64_t lda, bool transA, const double* B,
            int64_t ldb, bool transB, double* C, int64_t ldc) {
    if (M <= 0 || N <= 0) return;
    if (K <= 0) {
        for (int64_t i = 0; i < M; ++i)
            for (int64_t j = 0; j < N; ++j) C[i * ldc + j] = 0.0;
        return;
    }
    const Operand opA{A, lda, transA}, opB{B, ldb, transB};
    const int64_t mb = (M + MC - 1) / MC, nb = (N + NC - 1) / NC;
    // a task owns one MC x NC block of C and walks all K blocks in order
    parallel_for(mb * nb, [&](int64_t task) {
        const int64_t i0 = (task % mb) * MC, j0 = (task / mb) * NC;
        const int64_t mc = std::min(MC, M - i0), nc = std::min(NC, N - j0);
        const int64_t mpanels = (mc + MR - 1) / MR, npanels = (nc + NR - 1) / NR;
        std::vector<double> Ap(static_cast<size_t>(mpanels * MR * KC));
        std::vector<double> Bp(static_cast<size_t>(npanels * NR * KC));
        double edge[MR * NR];
        for (int64_t k0 = 0; k0 < K; k0 += KC) {
            const int64_t kc = std::min(KC, K - k0);
            const bool first = k0 == 0;
            pack_a(opA, i0, mc, k0, kc, Ap.data());
            pack_b(opB, j0, nc, k0, kc, Bp.data());
            for (int64_t q = 0; q < npanels; ++q) {
                const int64_t jj = j0 + q * NR;
                const int ncols = static_cast<int>(std::min<int64_t>(NR, j0 + nc - jj));
                for (int64_t p = 0; p < mpanels; ++p) {
                    const int64_t ii = i0 + p * MR;
                    const int nrows = static_cast<int>(std::min<int64_t>(MR, i0 + mc - ii));
                    const double* ap = Ap.data() + p * kc * MR;
                    const double* bp = Bp.data() + q * kc * NR;
                    if (nrows == MR && ncols == NR) {
                        tile(kc, ap, bp, C + ii * ldc + jj, ldc, first);
                        continue;
                    }
                    // ragged tile: run it on a full-size copy, keep the live part
                    for (int r = 0; r < MR; ++r)
                        for (int c = 0; c < NR; ++c)
                            edge[r * NR + c] = (r < nrows && c < ncols && !first) ? C[(ii + r) * ldc + jj + c] : 0.0;
                    tile(kc, ap, bp, edge, NR, first);
                    for (int r = 0; r < nrows; ++r)
                        for (int c = 0; c < ncols; ++c) C[(ii + r) * ldc + jj + c] = edge[r * NR + c];
                }
            }
        }
    });
}

}  // namespace oracle
