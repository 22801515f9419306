// fp64 C++ oracle of the MatrixFSDP owner-local optimizer step.
//
// TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the
// benchmark's host baseline load this library; the CUDA library never links,
// includes or calls it, and it includes nothing of the CUDA library.
//
// Method: "MatrixFSDP: communication-free matrix optimizers under ZeRO-3
// parameter sharding" (arxivlens summary page, Abstract; gist.science French
// summary, Methodologie sections 1-2).  Under owner-shaped placement the whole
// 2D weight and its full gradient sit on one data-parallel owner, which runs
// Muon (momentum-smoothed update, orthogonalised by Newton-Schulz) locally;
// non-matrix tensors are packed into a tail that stays on AdamW.  The pages
// name these steps without printing formulas; the arithmetic below is the
// standard Muon step with the Newton-Schulz definition fixed by the task:
//
//   1. buf <- beta buf + (1 - beta) G ;  M <- (1 - beta) G + beta buf   (Nesterov, EMA form)
//                                        M <- buf                       (plain momentum)
//   2. T = M^T when rows > cols, else M       (short side first; X is r x c, r <= c)
//   3. X_0 = T / (||T||_F + eps)
//   4. ns_steps times:  A = X X^T ;  B = b A + c (A A) ;  X <- a X + B X
//   5. O = (X_5 transposed back) * sqrt(max(1, rows / cols))
//   6. W <- W (1 - lr wd) - lr O
//
// and AdamW (decoupled decay, bias-corrected moments, step count t >= 1):
//   m <- beta1 m + (1 - beta1) g ;  v <- beta2 v + (1 - beta2) g^2
//   p <- p (1 - lr wd) - lr (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
//
// Everything is fp64 from the exact stored input values, in the order written
// above, with no blocking, fusion or reordering of the method's steps; the one
// primitive is the matrix product of matmul.cpp (ascending-k fused sums).
// Readings where the pages are silent (EMA Nesterov, eps = 1e-7 on the norm,
// strict rows > cols, the scale on the original shape, decay times lr on the
// pre-update W) are the same as the rest of this project's.
//
// The owner-segment form (oracle_muon_step_parts) takes the gradient as R
// ranks' contributions and sums them in rank order first: the owner receives
// exactly the full gradient (gist.science French summary, Methodologie
// section 2, owner-segment P2P collectives).
#include "oracle_f64.h"

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

constexpr int kOk = 0;
constexpr int kInvalid = -1;

struct MuonHp {
    double lr, beta, weight_decay, eps, a, b, c;
    int32_t ns_steps, nesterov;
};

struct AdamWHp {
    double lr, beta1, beta2, eps, weight_decay;
};

// rows of an r x c row-major matrix, split for the host threads
template <typename F>
void rows_parallel(int64_t r, F&& body) {
    const int64_t chunk = 64;
    oracle::parallel_for((r + chunk - 1) / chunk, [&](int64_t t) {
        const int64_t i1 = std::min(r, (t + 1) * chunk);
        for (int64_t i = t * chunk; i < i1; ++i) body(i);
    });
}

// Step 1.
void momentum(int64_t n, const double* G, const double* buf, double beta, int32_t nesterov, double* M,
              double* buf_out) {
    for (int64_t i = 0; i < n; ++i) {
        const double b = beta * buf[i] + (1.0 - beta) * G[i];
        buf_out[i] = b;
        M[i] = nesterov ? (1.0 - beta) * G[i] + beta * b : b;
    }
}

// Steps 2-4 and the transpose back: O = orthogonalised M (no shape scale).
void newton_schulz(int64_t rows, int64_t cols, const double* M, double a, double b, double c, int32_t steps,
                   double eps, double* O) {
    const bool tr = rows > cols;
    const int64_t r = tr ? cols : rows, cc = tr ? rows : cols;
    std::vector<double> X(static_cast<size_t>(r * cc));
    // step 2: X = T
    rows_parallel(r, [&](int64_t i) {
        for (int64_t j = 0; j < cc; ++j) X[i * cc + j] = tr ? M[j * cols + i] : M[i * cols + j];
    });
    // step 3: X_0 = T / (||T||_F + eps), the squares summed in row-major order of T
    double ss = 0.0;
    for (int64_t k = 0; k < r * cc; ++k) ss += X[k] * X[k];
    const double den = std::sqrt(ss) + eps;
    for (int64_t k = 0; k < r * cc; ++k) X[k] = X[k] / den;
    // step 4
    std::vector<double> A(static_cast<size_t>(r * r)), AA(static_cast<size_t>(r * r)), BX(static_cast<size_t>(r * cc));
    for (int32_t it = 0; it < steps; ++it) {
        oracle::matmul(r, r, cc, X.data(), cc, false, X.data(), cc, true, A.data(), r);        // A = X X^T
        oracle::matmul(r, r, r, A.data(), r, false, A.data(), r, false, AA.data(), r);        // A A
        rows_parallel(r, [&](int64_t i) {                                                    // B = b A + c (A A)
            for (int64_t j = 0; j < r; ++j) AA[i * r + j] = b * A[i * r + j] + c * AA[i * r + j];
        });
        oracle::matmul(r, cc, r, AA.data(), r, false, X.data(), cc, false, BX.data(), cc);    // B X
        rows_parallel(r, [&](int64_t i) {                                                    // X <- a X + B X
            for (int64_t j = 0; j < cc; ++j) X[i * cc + j] = a * X[i * cc + j] + BX[i * cc + j];
        });
    }
    // transpose back
    if (tr) {
        rows_parallel(rows, [&](int64_t i) {
            for (int64_t j = 0; j < cols; ++j) O[i * cols + j] = X[j * cc + i];
        });
    } else {
        std::memcpy(O, X.data(), sizeof(double) * static_cast<size_t>(r * cc));
    }
}

// Steps 1-6 for one matrix.
void muon_step(int64_t rows, int64_t cols, const double* W, const double* G, const double* buf, const MuonHp& hp,
               double* W_out, double* O_out, double* buf_out) {
    const int64_t n = rows * cols;
    std::vector<double> M(static_cast<size_t>(n));
    momentum(n, G, buf, hp.beta, hp.nesterov, M.data(), buf_out);
    if (n == 0) return;
    newton_schulz(rows, cols, M.data(), hp.a, hp.b, hp.c, hp.ns_steps, hp.eps, O_out);
    // step 5: the shape scale on the parameter's own (out, in) shape
    const double scale = std::sqrt(std::max(1.0, static_cast<double>(rows) / static_cast<double>(cols)));
    for (int64_t k = 0; k < n; ++k) O_out[k] = O_out[k] * scale;
    // step 6: decoupled weight decay and the write
    const double decay = 1.0 - hp.lr * hp.weight_decay;
    for (int64_t k = 0; k < n; ++k) W_out[k] = W[k] * decay - hp.lr * O_out[k];
}

bool valid(const MuonHp* hp) {
    return hp && hp->ns_steps >= 0 && (hp->nesterov == 0 || hp->nesterov == 1);
}

}  // namespace

extern "C" {

typedef MuonHp oracle_muon_hp;
typedef AdamWHp oracle_adamw_hp;

void oracle_set_threads(int32_t t) { oracle::set_threads(t); }
int32_t oracle_get_threads(void) { return oracle::threads(); }

int oracle_matmul(int64_t M, int64_t N, int64_t K, const double* A, int64_t lda, int32_t transA, const double* B,
                  int64_t ldb, int32_t transB, double* C, int64_t ldc) {
    if (M < 0 || N < 0 || K < 0) return kInvalid;
    if (M > 0 && N > 0 && (!C || (K > 0 && (!A || !B)))) return kInvalid;
    oracle::matmul(M, N, K, A, lda, transA != 0, B, ldb, transB != 0, C, ldc);
    return kOk;
}

int oracle_momentum(int64_t n, const double* G, const double* buf, double beta, int32_t nesterov, double* M_out,
                    double* buf_out) {
    if (n < 0 || (n > 0 && (!G || !buf || !M_out || !buf_out))) return kInvalid;
    momentum(n, G, buf, beta, nesterov, M_out, buf_out);
    return kOk;
}

int oracle_newton_schulz(int64_t rows, int64_t cols, const double* M, double a, double b, double c, int32_t steps,
                         double eps, double* O_out) {
    if (rows < 0 || cols < 0 || steps < 0) return kInvalid;
    if (rows == 0 || cols == 0) return kOk;
    if (!M || !O_out) return kInvalid;
    newton_schulz(rows, cols, M, a, b, c, steps, eps, O_out);
    return kOk;
}

int oracle_muon_step(int64_t rows, int64_t cols, const double* W, const double* G, const double* buf,
                     const oracle_muon_hp* hp, double* W_out, double* O_out, double* buf_out) {
    if (rows < 0 || cols < 0 || !valid(hp)) return kInvalid;
    if (rows * cols > 0 && (!W || !G || !buf || !W_out || !O_out || !buf_out)) return kInvalid;
    muon_step(rows, cols, W, G, buf, *hp, W_out, O_out, buf_out);
    return kOk;
}

// The owner's step on a gradient that arrives as nparts contributions:
// G = parts[0] + parts[1] + ... + parts[nparts-1], summed in that order.
int oracle_muon_step_parts(int64_t rows, int64_t cols, const double* W, const double* const* parts, int32_t nparts,
                           const double* buf, const oracle_muon_hp* hp, double* W_out, double* O_out,
                           double* buf_out) {
    if (rows < 0 || cols < 0 || nparts < 1 || !parts || !valid(hp)) return kInvalid;
    const int64_t n = rows * cols;
    if (n > 0 && (!W || !buf || !W_out || !O_out || !buf_out)) return kInvalid;
    for (int32_t q = 0; q < nparts; ++q)
        if (n > 0 && !parts[q]) return kInvalid;
    std::vector<double> G(static_cast<size_t>(n));
    for (int64_t k = 0; k < n; ++k) {
        double g = parts[0][k];
        for (int32_t q = 1; q < nparts; ++q) g = g + parts[q][k];
        G[k] = g;
    }
    muon_step(rows, cols, W, G.data(), buf, *hp, W_out, O_out, buf_out);
    return kOk;
}

// The owner's list of matrices, stepped one after another.
int oracle_muon_step_list(int32_t n, const int64_t* rows, const int64_t* cols, const double* const* W,
                          const double* const* G, const double* const* buf, const oracle_muon_hp* hp,
                          double* const* W_out, double* const* O_out, double* const* buf_out) {
    if (n < 0 || !valid(hp)) return kInvalid;
    if (n > 0 && (!rows || !cols || !W || !G || !buf || !W_out || !O_out || !buf_out)) return kInvalid;
    for (int32_t i = 0; i < n; ++i) {
        const int st = oracle_muon_step(rows[i], cols[i], W[i], G[i], buf[i], hp, W_out[i], O_out[i], buf_out[i]);
        if (st != kOk) return st;
    }
    return kOk;
}

int oracle_adamw_step(int64_t n, const double* p, const double* g, const double* m, const double* v, int64_t t,
                      const oracle_adamw_hp* hp, double* p_out, double* m_out, double* v_out) {
    if (n < 0 || t < 1 || !hp) return kInvalid;
    if (n > 0 && (!p || !g || !m || !v || !p_out || !m_out || !v_out)) return kInvalid;
    const double bc1 = 1.0 - std::pow(hp->beta1, static_cast<double>(t));
    const double bc2 = 1.0 - std::pow(hp->beta2, static_cast<double>(t));
    const double decay = 1.0 - hp->lr * hp->weight_decay;
    for (int64_t k = 0; k < n; ++k) {
        const double mk = hp->beta1 * m[k] + (1.0 - hp->beta1) * g[k];
        const double vk = hp->beta2 * v[k] + (1.0 - hp->beta2) * g[k] * g[k];
        const double m_hat = mk / bc1;
        const double v_hat = vk / bc2;
        p_out[k] = p[k] * decay - hp->lr * m_hat / (std::sqrt(v_hat) + hp->eps);
        m_out[k] = mk;
        v_out[k] = vk;
    }
    return kOk;
}

}  // extern "C"
