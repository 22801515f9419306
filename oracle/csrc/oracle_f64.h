// Internal declarations of the fp64 C++ oracle (test infrastructure only).
// Shared by the oracle's own sources; nothing of the CUDA library includes
// this file, and this file includes nothing of it.
#pragma once

#include <cstdint>
#include <functional>

namespace oracle {

// Number of host threads the oracle runs on (set by oracle_set_threads,
// default: the CPUs this process may run on).
int threads();
void set_threads(int t);   // t <= 0 restores the default

// Runs body(t) for t in [0, ntasks) on up to threads() host threads.  Tasks
// are independent; which thread runs a task does not change any result.
void parallel_for(int64_t ntasks, const std::function<void(int64_t)>& body);

// C = op(A) op(B) in fp64, C being M x N (row-major, leading dimension ldc).
//   op(A)[i][k] = transA ? A[k * lda + i] : A[i * lda + k]
//   op(B)[k][j] = transB ? B[j * ldb + k] : B[k * ldb + j]
// Every C[i][j] is the sum over k = 0, 1, ..., K-1, in that order, of the
// products op(A)[i][k] op(B)[k][j], each added with one fused multiply-add:
// acc <- fma(a_ik, b_kj, acc), acc starting at +0.  C must not overlap A or B.
void matmul(int64_t M, int64_t N, int64_t K, const double* A, int64_t lda, bool transA,
            const double* B, int64_t ldb, bool transB, double* C, int64_t ldc);

}  // namespace oracle
