// Internal declarations shared by the host dispatcher and the kernels of
// libmfsdp.  Nothing here crosses the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/mfsdp.h"

namespace mfsdp {

// Per-matrix record the kernels read from the workspace head.  X is the
// r x c working matrix (r <= c): M itself, or M^T when rows > cols.
struct MatDev {
    void*        param;       // W, rows x cols, param dtype
    const void*  grad;        // G, rows x cols, grad dtype
    float*       buf;         // momentum, rows x cols fp32
    float*       update_out;  // optional O, rows x cols fp32
    float*       xf[2];       // fp32 mode: fp32 X, ping-pong (unused in bf16 mode)
    __nv_bfloat16* xb[2];     // bf16 mode: hi part of X (the GEMM operand), ping-pong
    __nv_bfloat16* xlo[2];    // bf16 mode: lo part of X (master.cuh), ping-pong with xb
    float*       af;          // fp32 mode: E_A = A - diag(A), A = X X^T (r x r, zero diagonal)
    __nv_bfloat16* ab;        // bf16 mode: E_A in bf16 (GEMM operand and epilogue input)
    void*        bm;          // E_B = B - diag(B), B = b A + c A A: bf16 (bf16 mode) or fp32
    float*       da;          // diag(A), r entries, fp32
    float*       db;          // diag(B), r entries, fp32
    int64_t      rows, cols;  // the parameter's own shape
    int64_t      ldx;         // leading dimension (elements) of every X buffer
    int64_t      lda;         // leading dimension (elements) of A and B buffers
    int32_t      r, c;        // X shape
    int32_t      tr;          // rows > cols
    int32_t      param_bf16;
    int32_t      grad_bf16;
    int32_t      mom_flat;    // 1: the streaming kernels take this matrix as flat runs of
                              //    kFlatGroup elements (untransposed, rows a multiple of 8
                              //    elements, every user buffer 16-byte aligned); 0: as
                              //    groups of kMomGroup 64 x 64 tiles
    int32_t      mom_tiles_n; // momentum tiles along cols
    int32_t      mom_vec;     // 1: 16-byte vector access is legal for this matrix
    float        shape_scale; // sqrt(max(1, rows/cols))
    int32_t      mom_grp0;    // first group (one block of the streaming kernels) of this matrix
    int32_t      mom_groups_n;// groups of this matrix
    // owner-segment exchange (mfsdp_muon_step_p2p): the gradient is the fixed-order
    // sum of nparts contributions, and the updated parameter is also stored to
    // ncopies destinations; device arrays of pointers in the workspace head
    const void* const* gparts;
    void* const*       pcopies;
    int32_t      nparts;      // 0: the gradient is `grad`
    int32_t      ncopies;
};

// One output tile of a grouped GEMM phase.
struct TileDev {
    int32_t mat;
    int32_t tm;    // tile row index
    int32_t tn;    // tile column index
    int32_t kblk;  // K depth in units of the kernel's K block (scheduling weight)
};

// Diagonal-split form of one Newton-Schulz iteration.  With A = D_A + E_A and
// B = D_B + E_B (D diagonal, E zero-diagonal), the GEMMs take only the
// zero-diagonal parts as operands and the diagonals stay exact in fp32:
//   A A = E_A E_A + (d_i + d_j) E_A,ij + d_i^2 delta_ij
//   B X = E_B X + d_B,i X_ij
// In bf16 mode this keeps the large diagonal terms (and the near-cancellation
// a X + D_B X) out of bf16 rounding; the GEMM work is unchanged.
enum Phase : int32_t {
    PH_GRAM = 0,   // A = s^2 X X^T -> E_A, d_A          (upper tiles; tensor-core engine: block-upper
                   //                                      storage, the SIMT engine mirrors)
    PH_POLY = 1,   // B = b A + c A A -> E_B operand, d_B  (likewise)
    PH_APPLY = 2,  // X <- s ((a + d_B,i) X + E_B X)
    PH_FINAL = 3,  // the last iteration's X update (the same arithmetic); the parameter
                   // write then runs as its own HBM-bound kernel
};

struct StepScalars {
    float a, b, c;
    float lr;
    float decay;       // 1 - lr * wd
    float beta;
    float eps;
    int32_t nesterov;
    int32_t bf16_mode;
};

constexpr int kMomTile = 64;   // momentum / parameter-write tile: 64 x 64 elements of M or W
constexpr int kMomGroup = 4;   // tiles one block of those kernels processes
constexpr int kFlatGroup = kMomGroup * kMomTile * kMomTile;   // elements of a flat group (16384)

// The grouped step behind mfsdp_muon_step (segs == nullptr) and mfsdp_muon_step_p2p.
// always_upload: enqueue the descriptor-table upload on every call instead of
// skipping it when the workspace is known to hold the same table already (for a
// scratch that several matrix lists share).
int muon_step_impl(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                   const mfsdp_muon_hparams* hp, void* workspace, size_t workspace_bytes, void* stream,
                   bool always_upload = false);

// launch timing hooks (profile.cu): slot = prof_before(class, stream); launch; prof_after(slot, stream)
int prof_before(int cls, cudaStream_t s);
void prof_after(int slot, cudaStream_t s);

// device status word helpers (defined in status.cu)
int32_t* device_status_ptr();   // device address of this device's status word (nullptr on error)

// ---- launchers (return cudaError_t of the launch) ----
// parts: the gradients are owner-segment sums (MatDev::gparts) rather than MatDev::grad
// The streaming kernels run over groups: [0, flat_groups) belong to flat matrices
// (a flat-run kernel), [flat_groups, total_groups) to tiled ones (a 64 x 64 tile
// kernel); one launch each when non-empty.
// parts: the gradients are owner-segment sums (MatDev::gparts) rather than MatDev::grad
// flat_bulk: every flat matrix has bf16 gradients (momentum) or a bf16 parameter in bf16
// mode (parameter write), so its groups stream through 1D bulk copies
cudaError_t launch_momentum(const MatDev* d_mats, int32_t nmats, int32_t flat_groups, int32_t total_groups,
                            const StepScalars& sc, float* partials, bool parts, bool flat_bulk, cudaStream_t st);
cudaError_t launch_norm(const MatDev* d_mats, int32_t nmats, const float* partials,
                        float* s_out, float eps, cudaStream_t st);
// W <- W (1 - lr wd) - lr * scale * (use_s ? s : 1) * X, X from master copy xsel
// (bf16 mode: xb[xsel] + xlo[xsel]; fp32 mode: xf[xsel])
cudaError_t launch_param_write(const MatDev* d_mats, int32_t nmats, int32_t flat_groups, int32_t total_groups,
                               const StepScalars& sc, const float* s, int32_t xsel, int32_t use_s, bool flat_bulk,
                               cudaStream_t st);
cudaError_t launch_gemm_simt(Phase ph, const MatDev* d_mats, int32_t nmats, const TileDev* d_tiles, int32_t ntiles,
                             int32_t iter, const StepScalars& sc, const float* s, cudaStream_t st);
cudaError_t launch_adamw(float* p, const float* g, float* m, float* v, int64_t n,
                         float lr, float beta1, float beta2, float eps, float decay,
                         float bc1, float bc2, cudaStream_t st);

constexpr int kSimtTile = 128;  // SIMT GEMM block tile (square)

}  // namespace mfsdp
