/*
 * mfsdp.h - C ABI of the MatrixFSDP owner-local optimizer step on B200 (sm_100a).
 *
 * Method: "MatrixFSDP: communication-free matrix optimizers under ZeRO-3
 * parameter sharding" (arxivlens summary page, Abstract; gist.science French
 * and Portuguese technical summaries, Methodologie / Metodologia sections 1-2).
 * Under owner-shaped ZeRO-3 placement each 2D weight lives whole on one
 * data-parallel owner, so after the ordinary backward reduction the owner holds
 * the full gradient and runs the Muon update locally with no collective;
 * non-matrix tensors are packed into a tail that stays on AdamW.  This library
 * is that owner-local step, plus the host-side owner planner.
 *
 * Conventions shared by every entry point
 *  - Every call returns an int status: MFSDP_OK (0) or a negative MFSDP_ERR_*.
 *    No C++ exception crosses the ABI.  mfsdp_status_string() names a status.
 *  - Matrices are row-major, torch Linear layout: rows = out, cols = in.
 *  - Device pointers are plain CUDA device addresses on the current device;
 *    host pointers are ordinary host memory.  The caller owns every buffer;
 *    the library allocates no device memory and keeps no state across calls
 *    apart from a host-side cache of the descriptor table it last wrote into
 *    a given workspace (see mfsdp_muon_step).
 *  - "stream" is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  GPU work is enqueued asynchronously on it; arguments are
 *    validated synchronously before anything is enqueued, and an invalid call
 *    enqueues nothing.  Errors raised by kernels while they run are recorded
 *    in a device status word read by mfsdp_get_device_status().
 *  - A size of zero (n == 0, rows == 0 or cols == 0) is a no-op, not an error.
 */
#ifndef MFSDP_H
#define MFSDP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define MFSDP_OK                        0
#define MFSDP_ERR_INVALID_ARG          -1  /* NULL pointer, negative size, bad enum, aliasing */
#define MFSDP_ERR_UNSUPPORTED_DTYPE    -2  /* dtype/mode combination not implemented */
#define MFSDP_ERR_MISALIGNED           -3  /* pointer not aligned to its element size / 256 B workspace */
#define MFSDP_ERR_WORKSPACE_TOO_SMALL  -4  /* workspace_bytes below mfsdp_muon_workspace_size() */
#define MFSDP_ERR_CUDA                 -5  /* a CUDA runtime call failed (launch, copy, attribute) */
#define MFSDP_ERR_TIMEOUT              -6  /* a bounded device-side wait gave up */
#define MFSDP_ERR_DEVICE_FAULT         -7  /* a kernel detected an out-of-range index and skipped it */
#define MFSDP_ERR_UNSUPPORTED_DEVICE   -8  /* current device is not sm_100 */

/* ---- enums ----------------------------------------------------------- */
#define MFSDP_DTYPE_F32   0
#define MFSDP_DTYPE_BF16  1

#define MFSDP_KIND_MATRIX 0   /* 2D weight: Muon on its owner */
#define MFSDP_KIND_TAIL   1   /* non-matrix tensor: packed tail, AdamW */

#define MFSDP_MODE_FP32   0   /* Newton-Schulz GEMMs in fp32 on FFMA (no tf32) */
#define MFSDP_MODE_BF16   1   /* GEMM operands rounded to bf16, fp32 accumulate (tcgen05) */

/* ---- planner ----------------------------------------------------------
 * Passage: arxivlens summary page, Abstract (MatrixShard metadata, a
 * balance-aware owner planner, one owner per 2D weight with empty shards
 * elsewhere, non-matrix tensors packed into tail owners); gist.science French
 * summary, Methodologie section 2, "Metadonnees MatrixShard & Planificateur
 * Global" (owners balance resident bytes and optimizer work).
 */
typedef struct {
    int64_t rows;     /* >= 0; a 1D tensor of length L is rows = L, cols = 1 */
    int64_t cols;     /* >= 0 */
    int32_t kind;     /* MFSDP_KIND_MATRIX or MFSDP_KIND_TAIL */
    int32_t dtype;    /* MFSDP_DTYPE_* of a matrix's param and grad (tails are fp32) */
} mfsdp_param_desc;

/* One MatrixShard record: where a parameter lives and what it costs. */
typedef struct {
    int64_t param_id;        /* index into the planner's input array */
    int64_t rows, cols;
    int32_t owner;           /* owning rank in [0, world_size) */
    int32_t kind;            /* MFSDP_KIND_* */
    int32_t transposed;      /* 1 if rows > cols: Newton-Schulz runs on the transpose */
    int32_t reserved;
    double  ns_flops;        /* ns_steps * (4 r^2 c + 2 r^3), r = min, c = max; 0 for tails */
    int64_t resident_bytes;  /* param + grad + fp32 momentum (matrix) or 16 B/elem (tail) */
    int64_t owner_offset;    /* element offset in the owner's local buffer (matrices, id order)
                                or in the packed tail (tail tensors, id order) */
    double  shape_scale;     /* sqrt(max(1, rows / cols)); 1 for tails */
} mfsdp_matrix_shard;

/*
 * mfsdp_plan - assign an owner to every parameter (host only, no CUDA call).
 *   params          host array of n descriptors (read only)
 *   n               number of parameters, >= 0
 *   world_size      number of data-parallel ranks, >= 1
 *   ns_steps        Newton-Schulz iteration count used in the FLOP cost, >= 0
 *   out_shards      host array of n records, written (input order)
 *   out_rank_flops  host array of world_size doubles, written (may be NULL)
 *   out_rank_bytes  host array of world_size int64s, written (may be NULL)
 * Rule: matrices sorted by (-ns_flops, -resident_bytes, id); each goes to the
 * rank minimising (max((F_r+f)/Fbar, (B_r+b)/Bbar), F_r+f, rank); the whole
 * tail is one unit placed last on the rank with the fewest bytes.
 * Pure and deterministic.  Errors: MFSDP_ERR_INVALID_ARG.
 */
int mfsdp_plan(const mfsdp_param_desc* params, int64_t n, int32_t world_size, int32_t ns_steps,
               mfsdp_matrix_shard* out_shards, double* out_rank_flops, int64_t* out_rank_bytes);

/* The heaviest rank: largest FLOPs, then largest bytes, then lowest id. */
int mfsdp_heaviest_rank(const double* rank_flops, const int64_t* rank_bytes, int32_t world_size,
                        int32_t* out_rank);

/* ---- Owner-shard checkpoint resharding ----------------------------------
 * Passage: gist.science French summary, Methodologie section 2, "Checkpointing
 * et Routage" (and the Portuguese summary's Metodologia section 2): checkpoints
 * save the placement layout, the optimizer state is routed to its owners
 * through the MatrixShard metadata (Muon state for matrices, AdamW state for
 * tails), and a checkpoint can be restored on another world size.
 */

/* Where one parameter's checkpointed state goes.  The state is the parameter
 * and its fp32 momentum (matrix) or fp32 p, m, v (tail element); offsets are
 * in elements of the owner's local buffer (matrices, parameter-id order) or of
 * the packed tail, as in mfsdp_matrix_shard.owner_offset. */
typedef struct {
    int64_t param_id;
    int32_t kind;            /* MFSDP_KIND_MATRIX or MFSDP_KIND_TAIL */
    int32_t src_rank;        /* owner in the saved layout */
    int32_t dst_rank;        /* owner in the new layout */
    int32_t reserved;
    int64_t src_offset;
    int64_t dst_offset;
    int64_t elems;           /* rows * cols */
    int64_t state_bytes;     /* elems * (param bytes + 4) for a matrix, elems * 12 for a tail */
} mfsdp_reshard_route;

/*
 * mfsdp_reshard - plan the parameters of a saved layout for another world size
 * and route every parameter's state (host only, no CUDA call).
 *   params           host array of n descriptors, those the saved layout was planned from
 *   saved            host array of n MatrixShard records of the saved layout (any world size)
 *   n                number of parameters, >= 0
 *   new_world_size   >= 1
 *   ns_steps         as for mfsdp_plan
 *   out_shards       host array of n records, written: exactly mfsdp_plan(params, n, new_world_size, ns_steps)
 *   out_routes       host array of n routes, written in input order
 *   out_moved_bytes  state bytes of the parameters whose owner rank changes (may be NULL)
 * Pure and deterministic.  Errors: MFSDP_ERR_INVALID_ARG (a NULL array with
 * n > 0, a bad world size, a saved record whose id, shape or kind does not match
 * its descriptor, or a negative saved owner or offset), and the errors of mfsdp_plan.
 */
int mfsdp_reshard(const mfsdp_param_desc* params, const mfsdp_matrix_shard* saved, int64_t n,
                  int32_t new_world_size, int32_t ns_steps, mfsdp_matrix_shard* out_shards,
                  mfsdp_reshard_route* out_routes, int64_t* out_moved_bytes);

/* ---- Muon step --------------------------------------------------------
 * Passage: arxivlens summary page, Abstract (Muon orthogonalises
 * momentum-smoothed matrix updates with Newton-Schulz; the owner holds the
 * whole matrix, so Newton-Schulz runs locally); gist.science French summary,
 * Methodologie section 1 (the full gradient lands on the owner, which updates
 * with zero optimizer-step communication).  Arithmetic per matrix (fp32
 * unless stated):
 *   buf <- beta buf + (1-beta) G ;  M <- (1-beta) G + beta buf   (nesterov = 1)
 *                                   M <- buf                      (nesterov = 0)
 *   X <- (rows > cols ? M^T : M) / (||M||_F + eps)        (X is r x c, r <= c)
 *   ns_steps times:  A = X X^T ;  B = b A + c A A ;  X <- a X + B X
 *   O = (transpose back) X * sqrt(max(1, rows/cols))
 *   W <- W (1 - lr wd) - lr O        (one round-to-nearest-even store to W's dtype)
 * MFSDP_MODE_BF16 rounds the GEMM operands (X, A, B, without their diagonals)
 * to bf16 and accumulates in fp32; the diagonals of A and B and all epilogue
 * arithmetic stay fp32, and X is kept between iterations as bf16(X) plus
 * bf16(X - bf16(X)), within 2^-16 of X.  MFSDP_MODE_FP32 is fp32 throughout.
 */
typedef struct {
    void*       param;       /* device, rows x cols, param_dtype; updated in place */
    const void* grad;        /* device, rows x cols, grad_dtype; read only */
    float*      momentum;    /* device, rows x cols fp32 momentum buffer; updated in place */
    float*      update_out;  /* device, rows x cols fp32, optional (NULL = skip): receives O */
    int64_t     rows, cols;  /* >= 0 */
    int32_t     param_dtype; /* MFSDP_DTYPE_F32 or MFSDP_DTYPE_BF16 */
    int32_t     grad_dtype;  /* MFSDP_DTYPE_F32 or MFSDP_DTYPE_BF16 */
} mfsdp_matrix;

typedef struct {
    float   lr;              /* learning rate */
    float   beta;            /* momentum coefficient in [0, 1) */
    float   weight_decay;    /* decoupled, multiplied by lr */
    float   eps;             /* added to the Frobenius norm (1e-7) */
    float   a, b, c;         /* quintic coefficients (3.4445, -4.7750, 2.0315) */
    int32_t ns_steps;        /* Newton-Schulz iterations, 0..16 (5) */
    int32_t nesterov;        /* 1 = Nesterov, 0 = plain momentum */
    int32_t mode;            /* MFSDP_MODE_FP32 or MFSDP_MODE_BF16 */
} mfsdp_muon_hparams;

/*
 * mfsdp_muon_workspace_size - bytes of device workspace mfsdp_muon_step needs
 * for this matrix list and mode (host only).  *bytes is written.
 * Errors: MFSDP_ERR_INVALID_ARG, MFSDP_ERR_UNSUPPORTED_DTYPE.
 */
int mfsdp_muon_workspace_size(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                              size_t* bytes);

/*
 * mfsdp_muon_step - the owner's grouped Muon step over n matrices.
 *   mats             host array of n matrix records (read during the call only)
 *   hp               host pointer to the hyper-parameters
 *   workspace        device, >= mfsdp_muon_workspace_size() bytes, 256-byte aligned,
 *                    owned by the caller, dedicated to this matrix list: its head
 *                    holds a descriptor table the library writes on the first call
 *                    for a given (list, workspace) pair and reuses while the list
 *                    is unchanged.  Calls that share a workspace must not overlap
 *                    on the GPU.  Call mfsdp_muon_forget_workspace() before giving
 *                    the memory another use.
 *   stream           cudaStream_t as void*
 * Alignment: param/grad aligned to their element size, momentum and
 * update_out to 4 bytes (16-byte alignment enables vector access).  Matrices
 * must not alias one another.  Launches: the momentum kernel and the
 * parameter-write kernel once each for the flat matrices (untransposed, rows a
 * multiple of 8 elements, every buffer 16-byte aligned) and once each for the
 * others, one norm kernel, three GEMM-phase kernels per Newton-Schulz
 * iteration (mfsdp_muon_step_launches counts them).
 * Errors: MFSDP_ERR_INVALID_ARG, MFSDP_ERR_UNSUPPORTED_DTYPE, MFSDP_ERR_MISALIGNED,
 * MFSDP_ERR_WORKSPACE_TOO_SMALL, MFSDP_ERR_UNSUPPORTED_DEVICE, MFSDP_ERR_CUDA.
 */
int mfsdp_muon_step(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                    void* workspace, size_t workspace_bytes, void* stream);

/* ---- owner-segment exchange fused into the step -------------------------
 * Passage: arxivlens summary page, Abstract (deterministic owner-segment
 * collectives: the ordinary backward reduction lands the full gradient on
 * the owner, and forward/backward materialise parameters from the owner);
 * gist.science French summary, Methodologie section 2, "Collectifs P2P
 * Segment-Proprietaire" (gradient reduction writes only into the owner's
 * segment; materialisation moves only non-empty owner segments to the ranks
 * that need them).  mfsdp_muon_step_p2p is mfsdp_muon_step with both exchanges
 * done inside its kernels over plain device pointers, which may point into
 * peer GPUs' memory (NVLink / NVSwitch, with peer access enabled by the
 * caller or memory mapped through CUDA IPC):
 *   G = grad_parts[0] + grad_parts[1] + ... + grad_parts[nparts-1]
 *       (summed in that order in fp32 inside the momentum kernel; the
 *        matrix's own `grad` field is ignored and may be NULL)
 *   after the step, the updated parameter is also stored, bit for bit, to
 *   every param_copies[d] (inside the parameter-write kernel).
 */
#define MFSDP_MAX_PARTS  64
#define MFSDP_MAX_COPIES 64

typedef struct {
    const void* const* grad_parts;   /* host array of nparts device pointers, rows x cols of grad_dtype,
                                        each aligned to its element size; read only */
    void* const*       param_copies; /* host array of ncopies device pointers, rows x cols of param_dtype,
                                        aligned like param; written; NULL when ncopies = 0 */
    int32_t            nparts;       /* 1..MFSDP_MAX_PARTS */
    int32_t            ncopies;      /* 0..MFSDP_MAX_COPIES */
} mfsdp_owner_segments;

/* Workspace for mfsdp_muon_step_p2p (the descriptor table also holds the part
 * and copy pointers).  segs: host array of n records, one per matrix. */
int mfsdp_muon_workspace_size_p2p(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                                  const mfsdp_muon_hparams* hp, size_t* bytes);

/* The grouped step with the gradient reduction and the parameter
 * materialisation fused in (see above).  Same workspace rules, results and
 * errors as mfsdp_muon_step; the result does not depend on where the parts and
 * copies live.  Memory that aliases another matrix's buffers, or parts and
 * copies that overlap, are the caller's error (peer memory cannot be checked). */
int mfsdp_muon_step_p2p(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                        const mfsdp_muon_hparams* hp, void* workspace, size_t workspace_bytes, void* stream);

/* ---- owner-segment materialisation overlapped with the step ---------------
 * Passage: the same as mfsdp_muon_step_p2p (gist.science French summary,
 * Methodologie section 2, "Collectifs P2P Segment-Proprietaire": the owner
 * materialises its updated segments to the ranks that need them).  The step of
 * mfsdp_muon_step_p2p, split into `groups` contiguous groups of the list (in
 * list order, of about equal Newton-Schulz work), stepped one after another on
 * `stream`; as soon as a group's parameters are written, their copies to every
 * param_copies[d] are enqueued on `copy_stream` and run on the copy engines
 * while the later groups compute.  Before returning, the call makes `stream`
 * wait for every copy, so work enqueued on `stream` afterwards sees all of them.
 *   groups       1..64 (1: no overlap, the copies follow the whole step)
 *   copy_stream  cudaStream_t as void*, a stream other than `stream` for the
 *                overlap (NULL = the legacy default stream, which serialises)
 *   workspace    >= mfsdp_muon_workspace_size_p2p_overlap() bytes, 256-byte
 *                aligned: one region per group, each with the workspace rules of
 *                mfsdp_muon_step; call mfsdp_muon_forget_workspace_range() on the
 *                whole workspace before giving the memory another use
 * Results are bit for bit those of mfsdp_muon_step_p2p with the same arguments.
 * Errors: those of mfsdp_muon_step_p2p.
 */
int mfsdp_muon_workspace_size_p2p_overlap(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                                          const mfsdp_muon_hparams* hp, int32_t groups, size_t* bytes);

int mfsdp_muon_step_p2p_overlap(const mfsdp_matrix* mats, const mfsdp_owner_segments* segs, int32_t n,
                                const mfsdp_muon_hparams* hp, int32_t groups, void* workspace,
                                size_t workspace_bytes, void* stream, void* copy_stream);

/* Number of kernel launches one mfsdp_muon_step call with these arguments enqueues. */
int mfsdp_muon_step_launches(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp,
                             int32_t* launches);

/* Drop the host-side cache entry for a workspace (before reusing its memory). */
int mfsdp_muon_forget_workspace(void* workspace);

/* Drop every host-side cache entry for workspaces that start inside
 * [workspace, workspace + bytes): the per-group regions of a
 * mfsdp_muon_step_p2p_overlap workspace.  Errors: MFSDP_ERR_INVALID_ARG
 * (the range wraps around). */
int mfsdp_muon_forget_workspace_range(void* workspace, size_t bytes);

/*
 * mfsdp_muon_step_noalloc - mfsdp_muon_step without a caller workspace, for
 * callers that cannot allocate device memory at step time: hosts and plugins
 * that hand out every byte from their own pre-planned pools and forbid driver
 * allocations, and loops that must not enter an allocator (which may
 * synchronise the device).  The paper has no counterpart; this is a
 * deployment convenience of this library.
 *   mats, n, hp, stream  as for mfsdp_muon_step (same validation, same result)
 * Scratch: a fixed 64 MiB array compiled into the library, one per GPU that
 * loads it, held until process exit.  Lists whose mfsdp_muon_workspace_size()
 * exceeds 64 MiB are rejected with MFSDP_ERR_WORKSPACE_TOO_SMALL before any
 * GPU work.  The call allocates no device memory.
 * The first call on a device resolves the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  Every call shares the one array and keeps its
 * contents until the next call, so calls that overlap on the GPU (other
 * streams, other threads) race; serialise them.  Each call enqueues the upload
 * of its own descriptor and tile tables into the array on `stream` before its
 * kernels, and nothing else in the array needs to start at zero: every value
 * a call's results depend on is written by that call before it is read.
 */
int mfsdp_muon_step_noalloc(const mfsdp_matrix* mats, int32_t n, const mfsdp_muon_hparams* hp, void* stream);

/* ---- AdamW tail -------------------------------------------------------
 * Passage: arxivlens summary page, Abstract (non-matrix tensors are packed
 * into tail owners and stay on AdamW); gist.science French summary,
 * Methodologie section 1, "Tenseurs Non-Matrices".
 *   m <- beta1 m + (1-beta1) g ;  v <- beta2 v + (1-beta2) g^2
 *   p <- p (1 - lr wd) - lr (m / (1-beta1^t)) / (sqrt(v / (1-beta2^t)) + eps)
 */
typedef struct {
    float   lr, beta1, beta2, eps, weight_decay;
    int32_t reserved;
    int64_t step;            /* t >= 1, the step being taken */
} mfsdp_adamw_hparams;

/*
 * mfsdp_adamw_tail - AdamW over a flat packed fp32 tail of n elements.
 *   p, m, v  device fp32, updated in place;  g  device fp32, read only.
 *   All four 4-byte aligned, non-overlapping (16-byte alignment enables
 *   128-bit access).  Errors: MFSDP_ERR_INVALID_ARG, MFSDP_ERR_MISALIGNED,
 *   MFSDP_ERR_UNSUPPORTED_DEVICE, MFSDP_ERR_CUDA.
 */
int mfsdp_adamw_tail(float* p, const float* g, float* m, float* v, int64_t n,
                     const mfsdp_adamw_hparams* hp, void* stream);

/* ---- profiling ---------------------------------------------------------
 * Per-kernel-class CUDA-event timing of the library's own launches, for the
 * benchmark's roofline figures.  Between mfsdp_profile_begin() and
 * mfsdp_profile_end() every kernel the library launches (from any thread) is
 * bracketed by two cudaEventRecord calls on its launch stream, up to
 * max_launches launches; the rest run untimed.  mfsdp_profile_end()
 * synchronises those events, sums durations per class and stops recording.
 */
#define MFSDP_KCLASS_MOMENTUM  0   /* momentum + layout + norm partials */
#define MFSDP_KCLASS_NORM      1   /* Frobenius norm finalisation */
#define MFSDP_KCLASS_GRAM      2   /* A = X X^T */
#define MFSDP_KCLASS_POLY      3   /* B = b A + c A A */
#define MFSDP_KCLASS_APPLY     4   /* X <- a X + B X */
#define MFSDP_KCLASS_WRITE     5   /* parameter write: W <- W (1 - lr wd) - lr O */
#define MFSDP_KCLASS_ADAMW     6   /* AdamW tail */
#define MFSDP_KCLASS_FINAL     7   /* last iteration's X <- a X + B X (fp32 master only) */
#define MFSDP_KCLASS_COUNT     8

typedef struct {
    int32_t launches[MFSDP_KCLASS_COUNT];  /* timed launches per class */
    double  ms[MFSDP_KCLASS_COUNT];        /* summed device time per class, milliseconds */
} mfsdp_profile;

/* Start recording (max_launches >= 1 event pairs).  Errors: MFSDP_ERR_INVALID_ARG
 * (already recording or max_launches < 1), MFSDP_ERR_CUDA. */
int mfsdp_profile_begin(int32_t max_launches);

/* Stop recording and fill *out.  Errors: MFSDP_ERR_INVALID_ARG (not recording), MFSDP_ERR_CUDA. */
int mfsdp_profile_end(mfsdp_profile* out);

/* ---- status ------------------------------------------------------------ */

/* Synchronise `stream` and read (then clear) the device status word of the
 * current device: MFSDP_OK or the first MFSDP_ERR_* a kernel recorded. */
int mfsdp_get_device_status(void* stream, int32_t* status);

/* Failure-detection self-test: launches one CTA whose only wait (the same
 * bounded mbarrier wait the GEMM engine uses, on a barrier that nothing
 * arrives on) gives up after limit_ns (1e3..1e10) and records
 * MFSDP_ERR_TIMEOUT in the device status word; the kernel then returns
 * normally and the context stays usable.  Read the result with
 * mfsdp_get_device_status().  Errors: MFSDP_ERR_INVALID_ARG, MFSDP_ERR_CUDA,
 * MFSDP_ERR_UNSUPPORTED_DEVICE. */
int mfsdp_selftest_bounded_wait(int64_t limit_ns, void* stream);

/* Static text for a status code (never NULL). */
const char* mfsdp_status_string(int32_t status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t mfsdp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MFSDP_H */
