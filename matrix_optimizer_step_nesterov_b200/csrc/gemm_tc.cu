// tcgen05 / TMEM / TMA engine of the Newton-Schulz GEMM phases (bf16 operands,
// fp32 accumulate) for sm_100a.
//
// One persistent, warp-specialised kernel serves the three phases of an
// iteration (see internal.h for the diagonal-split form they compute):
//   PH_GRAM   C = X X^T      K = c   A: X rows (K-major)   B: X rows (K-major)   upper tiles
//   PH_POLY   C = E_A E_A    K = r   A: E_A rows           B: E_A rows           upper tiles
//   PH_APPLY  C = E_B X      K = r   A: E_B rows           B: X (MN-major)       all tiles
// Output tile 128 x 256 (one cta_group::1 MMA of M=128, N=256, K=16 per 32 B
// of K); K staged 64 deep (one 128-byte swizzle atom of bf16) through a
// 4-stage TMA ring; a double-buffered 2 x 256-column fp32 accumulator in TMEM
// lets the epilogue of one tile overlap the mainloop of the next.
//
// Warp roles (320 threads): warp 0 issues TMA loads, warp 1 owns TMEM and
// issues the MMAs (one elected lane), warps 2-9 run the epilogue, two per TMEM
// lane quadrant (32 rows), each on half of the tile's columns.  Every mbarrier wait is bounded: past the
// limit the waiting thread records MFSDP_ERR_TIMEOUT in the device status
// word, raises a CTA-wide abort flag and returns; the other roles see the flag
// in their own waits, the producer drains the loads it has in flight, and
// warp 1 frees TMEM before the CTA exits.
#include "gemm_tc.h"
#include "master.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <functional>
#include <mutex>
#include <queue>
#include <utility>
#include <vector>

namespace mfsdp {
namespace {

constexpr int BM = 128;          // rows of the output tile held by one CTA (TMEM lanes)
constexpr int BN = 256;          // tile cols (MMA N)
constexpr int BK = 64;           // K per stage: one 128 B swizzle atom of bf16
constexpr int A_BYTES = BM * BK * 2;            // 16 KiB per CTA per stage
constexpr int TMEM_COLS = 2 * BN;               // two fp32 accumulators
constexpr int NUM_EPI_WARPS = 8;                // two per TMEM lane quadrant, each half the columns
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
// epilogue staging, one 32 x kStgW-word buffer per epilogue warp: fp32 accumulators (APPLY,
// FINAL; 36-word rows make 16-byte writes along a row and 16-byte reads of 8-column runs
// conflict-free) or, in its first 32 x 20 words, bf16 result pairs (GRAM, POLY)
constexpr int kStgW = 36;
constexpr int STG_BYTES = NUM_EPI_WARPS * 32 * kStgW * 4;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait
constexpr uint32_t kSuspendHintNs = 200000u;                // one suspended try_wait: at most ~0.2 ms

// CTAs per MMA: 1 (cta_group::1, M = 128) or 2 (a cluster pair running
// cta_group::2 MMAs of M = 256; each CTA loads its own 128 rows of A and half
// of B, the MMA reads B across the pair, so each SM fetches 32 KiB instead
// of 48 KiB per 64-deep K block).
template <int CG>
struct TcCfg {
    static constexpr int B_ROWS = BN / CG;                      // B rows (N) this CTA loads
    static constexpr int STAGE_BYTES = A_BYTES + B_ROWS * BK * 2;
    static constexpr int STAGES = CG == 1 ? 4 : 5;
    static constexpr int TILE_M = BM * CG;                      // rows of a tile
    static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STG_BYTES + 1024 /*align slack*/ + 256 /*barriers*/;
};
constexpr int kCtaGroup = 2;      // the engine's configuration

// per-matrix TMA descriptors, stored in the workspace head (64-byte aligned)
// E_A and E_B are stored block-upper: only the 256 x 256 tiles (I, J) with
// I <= J are written, each in full.  An operand tile whose K block lies left of
// the diagonal tile is read through the transposed (MN-major) view of tile (J, I).
struct alignas(64) TcMaps {
    CUtensorMap xk[2];   // X bf16 operand, K-major view: dims {c, r}, box {64, 128}
    CUtensorMap xm[2];   // X bf16 operand, MN-major 3D view: dims {64, r, c/64}, box {64, 64, B_ROWS/64}
    CUtensorMap ea;      // E_A bf16, K-major view: dims {r, r}, box {64, 128}
    CUtensorMap eb;      // E_B bf16, K-major view: dims {r, r}, box {64, 128}
    CUtensorMap eat;     // E_A bf16, MN-major 3D view: dims {64, r, r/64}, box {64, 64, 2}
    CUtensorMap ebt;     // E_B bf16, MN-major 3D view: dims {64, r, r/64}, box {64, 64, 2}
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// The same test, but a thread whose phase is not complete yet is suspended
// until it completes or about `hint_ns` nanoseconds pass, instead of
// returning at once: a waiting thread issues nothing while it sleeps.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.b32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait.  Returns false when the CTA is aborting (flag raised here on
// timeout, or by another role).
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             int32_t* status, unsigned long long limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait_suspend(bar, parity, kSuspendHintNs)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit_ns) {
            *abort_flag = 1;
            if (status) atomicCAS(status, 0, -6 /* MFSDP_ERR_TIMEOUT */);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// 3D tiled TMA loads (two 64-element MN chunks of an MN-major operand in one instruction)
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
        : "memory");
}
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// TMA load of this CTA's share of a cta_group::2 operand; completion is
// counted on the barrier at `bar_cluster` (the leader CTA's).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster,
                                                 int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tc_mma2(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// arrive on the barrier at this offset in both CTAs of the pair once the
// issuing thread's prior cta_group::2 MMAs complete
__device__ __forceinline__ void tc_commit2_both(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(bar), "h"((uint16_t)0x3) : "memory");
}

__device__ __forceinline__ void tc_commit2_local(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   K-major operand:  rows 128 B apart, 8-row groups SBO = 1024 B apart (LBO unused).
//   MN-major operand: 64-element MN chunks LBO apart, 8-row K groups SBO = 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;                 // descriptor version (sm_100)
    d |= 2ull << 61;                 // SWIZZLE_128B
    return d;
}

// Instruction descriptor: D fp32, A/B bf16, A and B K- or MN-major, N = 256, M = 128 or 256.
__host__ __device__ constexpr uint32_t make_idesc(bool a_mn_major, bool b_mn_major, int m) {
    return (1u << 4)                 // D format: F32
         | (1u << 7)                 // A format: BF16
         | (1u << 10)                // B format: BF16
         | ((a_mn_major ? 1u : 0u) << 15)
         | ((b_mn_major ? 1u : 0u) << 16)
         | (static_cast<uint32_t>(BN >> 3) << 17)
         | (static_cast<uint32_t>(m >> 4) << 24);
}

// ---------------------------------------------------------------------------
// Epilogues.  Each epilogue warp owns 32 accumulator rows (its TMEM lane
// quadrant) and 128 of the tile's 256 columns, in chunks of 32 x 32 read with
// tcgen05.ld.  TMEM delivers a chunk in the row domain: lane l holds row
// gi0 + l, columns gj0 .. gj0 + 31.  Accesses that run along a column (the
// mirrored triangle of a symmetric result) are issued straight from the row
// domain, where the 32 lanes touch 32 consecutive elements.  Accesses that run
// along a row go through the warp's 32 x 33 staging buffer into the column
// domain (lane l takes column gj0 + l, rows one by one), so they are coalesced
// too.  Every global input is loaded one half chunk (16 rows or columns) ahead
// of its use, and a tile's first half is loaded before the accumulator is
// ready, while the MMAs still run.
// ---------------------------------------------------------------------------

// GRAM / POLY input of half chunk b of chunks [q0, ..): POLY's E_A(gi, gj) for
// the 16 columns gj of the half, gj > gi, and d_A of those 16 columns (the same
// for every lane: broadcast loads).
//   off-diagonal tile: the tile's own elements E_A[gi][gj], 16 consecutive
//     elements of this lane's row (two 16-byte loads);
//   diagonal tile: the mirrored elements E_A[gj][gi], consecutive across lanes
//     (the diagonal tile is stored with both triangles).
template <int ph>
__device__ __forceinline__ void sym_load_half(const MatDev& md, bool offdiag, int gi, int gj_tile, int q0, int b,
                                              int Mrows, int Ncols, unsigned short (&ev)[16], float4 (&dq)[4]) {
    if (ph != PH_POLY) return;
    const unsigned short* ab = reinterpret_cast<const unsigned short*>(md.ab);
    const int64_t lda = md.lda;
    const int gjh = gj_tile + (q0 + (b >> 1)) * 32 + (b & 1) * 16;
    const bool row_ok = gi < Mrows;
    if (offdiag) {
        if (row_ok && gjh + 16 <= Ncols) {
            const uint4* p = reinterpret_cast<const uint4*>(ab + (int64_t)gi * lda + gjh);   // 16-byte aligned
            const uint4 u0 = __ldg(p), u1 = __ldg(p + 1);
            const uint32_t w[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
            #pragma unroll
            for (int k = 0; k < 8; ++k) {
                ev[2 * k] = static_cast<unsigned short>(w[k] & 0xFFFFu);
                ev[2 * k + 1] = static_cast<unsigned short>(w[k] >> 16);
            }
        } else {
            #pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int gj = gjh + k;
                ev[k] = (row_ok && gj < Ncols) ? __ldg(ab + (int64_t)gi * lda + gj) : (unsigned short)0;
            }
        }
    } else {
        #pragma unroll
        for (int k = 0; k < 16; ++k) {
            const int gj = gjh + k;
            ev[k] = (row_ok && gj < Ncols && gi < gj) ? __ldg(ab + (int64_t)gj * lda + gi) : (unsigned short)0;
        }
    }
    if (gjh + 16 <= Ncols) {
        const float4* p = reinterpret_cast<const float4*>(md.da + gjh);   // 16-byte aligned (gjh % 16 == 0)
        #pragma unroll
        for (int k = 0; k < 4; ++k) dq[k] = __ldg(p + k);
    } else {
        float d[16];
        #pragma unroll
        for (int k = 0; k < 16; ++k) d[k] = (gjh + k < Ncols) ? __ldg(md.da + gjh + k) : 0.f;
        #pragma unroll
        for (int k = 0; k < 4; ++k) dq[k] = make_float4(d[4 * k], d[4 * k + 1], d[4 * k + 2], d[4 * k + 3]);
    }
}

__device__ __forceinline__ float f4_elem(const float4 (&q)[4], int k) {
    const float4 v = q[k >> 2];
    return (k & 3) == 0 ? v.x : (k & 3) == 1 ? v.y : (k & 3) == 2 ? v.z : v.w;
}

// GRAM / POLY epilogue of one warp over its live chunks [q0, q1):
//   GRAM: A = s^2 acc  ->  E_A (bf16), d_A
//   POLY: B = b A + c A A with A A = acc + (d_i + d_j) E_A + d_i^2 delta_ij
//         ->  E_B (bf16), d_B
// Results are stored block-upper: an off-diagonal tile (I < J) writes only
// itself; a diagonal tile writes its upper triangle and mirrors it into its
// lower triangle.  The row-domain values go to the warp's staging buffer as the
// bf16 pairs the column-domain stores write (32 rows of 20 words: 16 pairs and
// 4 words of padding, so 16-byte writes and 4-byte reads are conflict-free).
// ev / dq hold the first half chunk's inputs, loaded by the caller.
template <int ph>
__device__ __forceinline__ void epilogue_sym_warp(const MatDev& md, const StepScalars& sc, float sg, bool offdiag,
                                                  int gi0, int gj_tile, int q0, int q1, int Mrows, int Ncols,
                                                  uint32_t trow, float (*stg)[kStgW], int lane, unsigned short (&ev)[16],
                                                  float4 (&dq)[4]) {
    constexpr int kSw = 20;                 // staging words per row
    uint32_t* sb = reinterpret_cast<uint32_t*>(&stg[0][0]);   // [32][kSw] words (2560 of the buffer's 4608 bytes)
    const int gi = gi0 + lane;      // row domain: this lane's row
    const bool row_ok = gi < Mrows;
    const int64_t lda = md.lda;
    __nv_bfloat16* ob = (ph == PH_GRAM) ? md.ab : static_cast<__nv_bfloat16*>(md.bm);
    const float di = (ph == PH_POLY && row_ok) ? __ldg(md.da + gi) : 0.f;
    const float s2 = sg * sg;
    unsigned short en[16];
    float4 dqn[4];
    const int nb = 2 * (q1 - q0);
    #pragma unroll 1
    for (int q = q0; q < q1; ++q) {
        const int gj0 = gj_tile + q * 32;
        uint32_t r[32];
        tmem_ld32(trow + q * 32, r);              // warp-collective
        // warp-uniform: the whole 32 x 32 chunk is inside the matrix and strictly above the diagonal
        const bool interior = gi0 + 31 < Mrows && gj0 + 31 < Ncols && gi0 + 31 < gj0;
        #pragma unroll
        for (int hh = 0; hh < 2; ++hh) {          // the chunk's two halves (h known at compile time)
            const int h = hh * 16;
            const int b = 2 * (q - q0) + hh;
            if (b + 1 < nb) sym_load_half<ph>(md, offdiag, gi, gj_tile, q0, b + 1, Mrows, Ncols, en, dqn);
            // element k of the half: its value, with the diagonal tile's mirror and the
            // diagonal entries stored on the way
            auto elem_in = [&](int k) -> float {   // interior chunks: strictly above the diagonal, inside
                const float acc = __uint_as_float(r[h + k]);
                float v;
                if (ph == PH_GRAM) {
                    v = s2 * acc;
                } else {
                    const float e = bf16_bits_to_float(ev[k]);
                    v = sc.b * e + sc.c * fmaf(di + f4_elem(dq, k), e, acc);
                }
                if (!offdiag) ob[(int64_t)(gj0 + h + k) * lda + gi] = __float2bfloat16_rn(v);   // mirror
                return v;
            };
            auto elem_edge = [&](int k) -> float {
                const float acc = __uint_as_float(r[h + k]);
                const int gj = gj0 + h + k;
                float v = 0.f;
                if (row_ok && gj < Ncols && gi <= gj) {
                    if (ph == PH_GRAM) {
                        v = s2 * acc;
                        if (gi == gj) {
                            md.da[gi] = v;
                            ob[(int64_t)gi * lda + gi] = __float2bfloat16_rn(0.f);
                        } else if (!offdiag) {
                            ob[(int64_t)gj * lda + gi] = __float2bfloat16_rn(v);   // lower triangle, along column gj
                        }
                    } else {
                        if (gi == gj) {
                            md.db[gi] = sc.b * di + sc.c * fmaf(di, di, acc);
                            ob[(int64_t)gi * lda + gi] = __float2bfloat16_rn(0.f);
                        } else {
                            const float e = bf16_bits_to_float(ev[k]);
                            v = sc.b * e + sc.c * fmaf(di + f4_elem(dq, k), e, acc);
                            if (!offdiag) ob[(int64_t)gj * lda + gi] = __float2bfloat16_rn(v);
                        }
                    }
                }
                return v;
            };
            // each bf16 pair is packed as soon as both of its values exist
            uint32_t pk[8];
            if (interior) {
                #pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const __nv_bfloat162 v2 = __floats2bfloat162_rn(elem_in(2 * k), elem_in(2 * k + 1));
                    pk[k] = *reinterpret_cast<const uint32_t*>(&v2);
                }
            } else {
                #pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const __nv_bfloat162 v2 = __floats2bfloat162_rn(elem_edge(2 * k), elem_edge(2 * k + 1));
                    pk[k] = *reinterpret_cast<const uint32_t*>(&v2);
                }
            }
            uint4* srow = reinterpret_cast<uint4*>(sb + lane * kSw + hh * 8);
            srow[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            srow[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
            #pragma unroll
            for (int k = 0; k < 16; ++k) ev[k] = en[k];
            #pragma unroll
            for (int k = 0; k < 4; ++k) dq[k] = dqn[k];
        }
        __syncwarp();
        // column domain: the upper-triangle copies (row gi0 + rr < column gjc)
        const int gjc = gj0 + lane;
        if (interior) {
            // two adjacent columns per lane and two rows per instruction: 4-byte stores
            const int cp = lane & 15, rp = lane >> 4;
            uint32_t* pu = reinterpret_cast<uint32_t*>(ob + (int64_t)gi0 * lda + gj0) + cp;
            const int64_t ldw = lda >> 1;             // lda is a multiple of 8
            #pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int rr = 2 * k + rp;
                pu[(int64_t)rr * ldw] = sb[rr * kSw + cp];
            }
        } else {
            const bool col_ok = gjc < Ncols;
            const __nv_bfloat16* sh = reinterpret_cast<const __nv_bfloat16*>(sb);   // element (rr, c) at rr * 2 kSw + c
            #pragma unroll 1
            for (int rr = 0; rr < 32; ++rr) {
                const int gi2 = gi0 + rr;
                if (gi2 < Mrows && col_ok && gi2 < gjc) ob[(int64_t)gi2 * lda + gjc] = sh[rr * 2 * kSw + lane];
            }
        }
        __syncwarp();
    }
}

// APPLY / FINAL input of one quarter chunk (8 rows of a 32 x 32 chunk): the hi
// and lo parts of X (master.cuh), copy `cur`, as 16-byte vectors.  Lane l takes
// row `row` and the 8 columns from `col` = 8 (l & 3) of the chunk, so a warp
// covers 8 rows of 32 columns.  (A vector may reach up to 7 columns past the
// matrix: into the padding of the leading dimension, whose values only ever
// reach discarded outputs.)
__device__ __forceinline__ void x_load8(const MatDev& md, int cur, int row, int col, int Mrows, int Ncols, uint4& h,
                                        uint4& l) {
    if (row < Mrows && col < Ncols) {
        const int64_t i = (int64_t)row * md.ldx + col;   // col and ldx multiples of 8: 16-byte aligned
        h = __ldg(reinterpret_cast<const uint4*>(md.xb[cur] + i));
        l = __ldg(reinterpret_cast<const uint4*>(md.xlo[cur] + i));
    } else {
        h = make_uint4(0u, 0u, 0u, 0u);
        l = h;
    }
}

// One whole chunk (its four quarters) of X for this lane: rows gi0 + (lane / 4) + 8k,
// the 8 columns from col.
__device__ __forceinline__ void x_load_chunk(const MatDev& md, int cur, int gi0, int col, int lane, int Mrows,
                                             int Ncols, uint4 (&h)[4], uint4 (&l)[4]) {
    #pragma unroll
    for (int k = 0; k < 4; ++k) x_load8(md, cur, gi0 + (lane >> 2) + 8 * k, col, Mrows, Ncols, h[k], l[k]);
}

// APPLY / FINAL epilogue of one warp over its live chunks [q0, q1):
//   X <- s ((a + d_B,i) X + E_B X)
// X is read from copy iter & 1 (hi and lo parts, through the read-only path)
// and written to the other copy, 8 elements (16 bytes of each part) per lane
// and access.  The loads run a whole chunk ahead of their use (ch / cl hold
// the first chunk, loaded by the caller while the MMAs still run).
template <bool S0>   // the first iteration: the Frobenius scale s applies (sg = s); later ones skip the product
__device__ __forceinline__ void epilogue_x_warp(const MatDev& md, int iter, const StepScalars& sc, float sg,
                                                int gi0, int gj_tile, int q0, int q1, int Mrows, int Ncols,
                                                uint32_t trow, float (*stg)[kStgW], int lane, uint4 (&ch)[4],
                                                uint4 (&cl)[4]) {
    const int cur = iter & 1;
    __nv_bfloat16* __restrict__ xhn = md.xb[cur ^ 1];
    __nv_bfloat16* __restrict__ xlon = md.xlo[cur ^ 1];
    const int64_t ldx = md.ldx;
    const int gi = gi0 + lane;
    const float fa = gi < Mrows ? (sc.a + __ldg(md.db + gi)) : 0.f;   // row domain: (a + d_B) of row gi
    const int cq = lane & 3, r8 = lane >> 2;
    #pragma unroll 1
    for (int q = q0; q < q1; ++q) {
        uint32_t r[32];
        tmem_ld32(trow + q * 32, r);              // warp-collective
        __syncwarp();                             // previous chunk's reads of stg are done
        #pragma unroll
        for (int t = 0; t < 32; t += 4)
            *reinterpret_cast<float4*>(&stg[lane][t]) = make_float4(__uint_as_float(r[t]), __uint_as_float(r[t + 1]),
                                                                    __uint_as_float(r[t + 2]), __uint_as_float(r[t + 3]));
        __syncwarp();
        uint4 nh[4], nl[4];
        if (q + 1 < q1) {
            x_load_chunk(md, cur, gi0, gj_tile + (q + 1) * 32 + 8 * cq, lane, Mrows, Ncols, nh, nl);
        } else {
            #pragma unroll
            for (int k = 0; k < 4; ++k) nh[k] = nl[k] = make_uint4(0u, 0u, 0u, 0u);
        }
        const int col = gj_tile + q * 32 + 8 * cq;
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int rr = r8 + 8 * k;            // row within the chunk
            const float fk = __shfl_sync(0xffffffffu, fa, rr);
            if (gi0 + rr < Mrows && col < Ncols) {
                const uint32_t hw[4] = {ch[k].x, ch[k].y, ch[k].z, ch[k].w}, lw[4] = {cl[k].x, cl[k].y, cl[k].z, cl[k].w};
                const float4 a0 = *reinterpret_cast<const float4*>(&stg[rr][8 * cq]);
                const float4 a1 = *reinterpret_cast<const float4*>(&stg[rr][8 * cq + 4]);
                const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
                uint32_t oh[4], ol[4];
                #pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float x0 = master_value(static_cast<uint16_t>(hw[j] & 0xFFFFu), static_cast<uint16_t>(lw[j] & 0xFFFFu));
                    const float x1 = master_value(static_cast<uint16_t>(hw[j] >> 16), static_cast<uint16_t>(lw[j] >> 16));
                    const float v0 = S0 ? sg * fmaf(fk, x0, av[2 * j]) : fmaf(fk, x0, av[2 * j]);
                    const float v1 = S0 ? sg * fmaf(fk, x1, av[2 * j + 1]) : fmaf(fk, x1, av[2 * j + 1]);
                    master_split2(v0, v1, oh[j], ol[j]);
                }
                const int64_t i = (int64_t)(gi0 + rr) * ldx + col;
                *reinterpret_cast<uint4*>(xhn + i) = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                *reinterpret_cast<uint4*>(xlon + i) = make_uint4(ol[0], ol[1], ol[2], ol[3]);
            }
        }
        #pragma unroll
        for (int k = 0; k < 4; ++k) {
            ch[k] = nh[k];
            cl[k] = nl[k];
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// the persistent kernel
// ---------------------------------------------------------------------------
// Which operands come from block-upper E storage: A of POLY, APPLY and FINAL
// (E_A, E_B) and B of POLY (E_A).
template <int ph>
constexpr bool kSymA = ph == PH_POLY || ph == PH_APPLY || ph == PH_FINAL;
template <int ph>
constexpr bool kSymB = ph == PH_POLY;

// Tiles come from a host-built table partitioned per cluster: cluster k runs
// tiles[seg[k]] .. tiles[seg[k + 1] - 1] in that order (every role of both
// CTAs walks the same segment).
template <int ph, int CG>
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_phase_kernel(const MatDev* __restrict__ mats, const TcMaps* __restrict__ maps, int32_t nmats,
                const TileDev* __restrict__ tiles, const int32_t* __restrict__ seg, int32_t iter, int32_t ring,
                StepScalars sc, const float* __restrict__ s, int32_t* status) {
    using C = TcCfg<CG>;
    constexpr int STAGES = C::STAGES;
    // stages of the ring this launch cycles through (the host's choice, at most the STAGES allocated)
    const int nst = (ring >= 2 && ring <= STAGES) ? ring : STAGES;
    constexpr int STAGE_BYTES = C::STAGE_BYTES;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned stage ring (128 B swizzle atoms need 1024 B alignment)
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* stg_all = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + STG_BYTES);
    // bars: full[STAGES], empty[STAGES], tmem_full[2], tmem_empty[2], mma_done
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
    const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
    const uint32_t mma_done = smem_u32(bars + 2 * STAGES + 4);
    const uint32_t rank = (CG == 2) ? cluster_rank() : 0u;      // 0 = leader (issues the MMAs)
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x / CG;
    const int t_begin = seg[cluster_id], t_end = seg[cluster_id + 1];

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(full0 + 8 * i, 1);
            mbar_init(empty0 + 8 * i, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull0 + 8 * i, 1);
            mbar_init(tempty0 + 8 * i, CG * NUM_EPI_WARPS);   // one arrive per epilogue warp of the pair
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        if (CG == 2) {
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                         ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();     // the peer's barriers are initialised before anyone signals them
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // Programmatic dependent launch: the set-up above may overlap the previous
    // phase's last tiles; nothing an earlier kernel wrote is read before this wait.
    // The next phase may then launch as soon as every CTA of this one has started.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    constexpr bool gemm = (ph == PH_APPLY || ph == PH_FINAL);
    const int cur = iter & 1;

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int issued[STAGES];                  // parity of the last fill issued per stage, -1 = none
            #pragma unroll
            for (int i = 0; i < STAGES; ++i) issued[i] = -1;
            for (int t = t_begin; t < t_end && ok; ++t) {
                const TileDev td = tiles[t];
                const MatDev& md = mats[td.mat];
                const TcMaps& mp = maps[td.mat];
                const int K = (ph == PH_GRAM) ? md.c : md.r;
                const int nk = (K + BK - 1) / BK;
                const CUtensorMap* amap = (ph == PH_GRAM) ? &mp.xk[cur] : (ph == PH_POLY) ? &mp.ea : &mp.eb;
                const CUtensorMap* bmap = (ph == PH_GRAM) ? &mp.xk[cur] : (ph == PH_POLY) ? &mp.ea : &mp.xm[cur];
                const CUtensorMap* amap_t = (ph == PH_POLY) ? &mp.eat : &mp.ebt;   // A of POLY / APPLY
                const int i0 = td.tm * C::TILE_M + (int)rank * BM;        // this CTA's A rows
                const int jb = td.tn * BN + (int)rank * C::B_ROWS;        // this CTA's share of B
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bounded(empty0 + 8 * stage, phase ^ 1, abort_flag, status)) { ok = false; break; }
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    const uint32_t fb = full0 + 8 * stage;
                    // block-upper storage: K blocks left of the operand's own diagonal tile
                    // come from the transposed tile
                    const int kt = kb / (BN / BK);
                    const bool a_t = kSymA<ph> && kt < td.tm;
                    const bool b_t = kSymB<ph> && kt < td.tn;
                    // a diagonal tile of GRAM or POLY: this CTA's B rows are its A rows, in the
                    // same view, so B is not loaded and the MMA reads it from the A buffer
                    const bool diag = !gemm && td.tm == td.tn;
                    const uint32_t bytes = diag ? A_BYTES : STAGE_BYTES;
                    if (CG == 1) mbar_arrive_expect_tx(fb, bytes);
                    else if (leader) mbar_arrive_expect_tx(fb, CG * bytes);   // both CTAs' bytes
                    const uint32_t fbl = (CG == 2) ? map_to_rank(fb, 0) : fb;
                    auto load = [&](uint32_t dst, const CUtensorMap* map, int x, int y) {
                        if (CG == 2) tma_load_2d_pair(dst, map, fbl, x, y);
                        else tma_load_2d(dst, map, fbl, x, y);
                    };
                    auto load3 = [&](uint32_t dst, const CUtensorMap* map, int chunk, int k) {
                        if (CG == 2) tma_load_3d_pair(dst, map, fbl, 0, k, chunk);
                        else tma_load_3d(dst, map, fbl, 0, k, chunk);
                    };
                    if (a_t) {
                        load3(sa, amap_t, i0 / 64, kb * BK);         // A rows i0 .. i0 + 127, MN-major
                    } else {
                        load(sa, amap, kb * BK, i0);
                    }
                    if (diag) {
                        // B comes from the A buffer (see above)
                    } else if (gemm || b_t) {
                        const CUtensorMap* bm_ = gemm ? bmap : &mp.eat;
                        load3(sb, bm_, jb / 64, kb * BK);            // B rows jb .. jb + B_ROWS - 1, MN-major
                    } else {
                        #pragma unroll
                        for (int h = 0; h < C::B_ROWS / 128; ++h) load(sb + h * (128 * BK * 2), bmap, kb * BK, jb + 128 * h);
                    }
                    issued[stage] = static_cast<int>(phase);
                    if (++stage == nst) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && leader) {
                // aborting: wait (bounded, 10 ms each) until every issued load has landed
                for (int i = 0; i < STAGES; ++i) {
                    if (issued[i] < 0) continue;
                    const unsigned long long t0 = globaltimer();
                    while (!mbar_try_wait(full0 + 8 * i, static_cast<uint32_t>(issued[i])) &&
                           globaltimer() - t0 < 10000000ull) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader CTA) ----------------
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = t_begin; t < t_end && ok; ++t) {
                const TileDev td = tiles[t];
                const MatDev& md = mats[td.mat];
                const int K = (ph == PH_GRAM) ? md.c : md.r;
                const int nk = (K + BK - 1) / BK;
                if (!wait_bounded(tempty0 + 8 * acc, acc_phase ^ 1, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < nk; ++kb) {
                    if (!wait_bounded(full0 + 8 * stage, phase, abort_flag, status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
                    const uint32_t sb = (!gemm && td.tm == td.tn) ? sa : sa + A_BYTES;   // the producer's diagonal case
                    const int kt = kb / (BN / BK);
                    const bool a_t = kSymA<ph> && kt < td.tm;           // same choice as the producer's
                    const bool b_t = gemm || (kSymB<ph> && kt < td.tn);
                    const uint32_t idesc = make_idesc(a_t, b_t, C::TILE_M);
                    #pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // K-major: 16 K columns = 32 B further along each row; MN-major: 16 K rows
                        // of 128 B further, 64-wide MN chunks BK * 128 B apart
                        const uint64_t ad = a_t ? smem_desc(sa + kk * 16 * 128, BK * 128, 1024)
                                                : smem_desc(sa + kk * 32, 16, 1024);
                        const uint64_t bd = b_t ? smem_desc(sb + kk * 16 * 128, BK * 128, 1024)
                                                : smem_desc(sb + kk * 32, 16, 1024);
                        if (CG == 2) tc_mma2(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                        else tc_mma(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    // stage free (in both CTAs) once these MMAs finish
                    if (CG == 2) tc_commit2_both(empty0 + 8 * stage);
                    else tc_commit(empty0 + 8 * stage);
                    if (++stage == nst) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                // accumulator ready for the epilogue (of both CTAs)
                if (CG == 2) tc_commit2_both(tfull0 + 8 * acc);
                else tc_commit(tfull0 + 8 * acc);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
            // every MMA this thread issued has completed before TMEM is freed (bounded)
            if (CG == 2) tc_commit2_local(mma_done);
            else tc_commit(mma_done);
            const unsigned long long t0 = globaltimer();
            while (!mbar_try_wait(mma_done, 0) && globaltimer() - t0 < 100000000ull) {
            }
        }
    } else {
        // ---------------- epilogue (warps 2..9, both CTAs) ----------------
        const int quad = warp & 3;                 // TMEM lane quadrant this warp may access
        const int half = (warp - 2) >> 2;          // which 128 of the tile's 256 columns
        const uint32_t tempty_leader0 = (CG == 2) ? map_to_rank(tempty0, 0) : tempty0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = t_begin; t < t_end; ++t) {
            const TileDev td = tiles[t];
            const MatDev md = mats[td.mat];   // a register copy: global stores below cannot alias it
            const int Mrows = md.r;
            const int Ncols = gemm ? md.c : md.r;
            const int gi0 = td.tm * C::TILE_M + (int)rank * BM + quad * 32;
            const int gj_tile = td.tn * BN;
            // this warp's live chunks [q0, q1): columns in range and (symmetric
            // phases) not entirely below the diagonal
            int q0 = half * (BN / 64);
            const int qb = q0 + BN / 64;
            if (!gemm)
                while (q0 < qb && gj_tile + q0 * 32 + 31 < gi0) ++q0;
            int q1 = q0;
            while (q1 < qb && gj_tile + q1 * 32 < Ncols) ++q1;
            const bool live = gi0 < Mrows && q0 < q1;
            // the first half chunk's inputs, loaded while the MMAs still run
            unsigned short pre_e[16];
            uint4 pre_h[4], pre_l[4];
            float4 pre_dq[4];
            if (live) {
                if constexpr (gemm)
                    x_load_chunk(md, iter & 1, gi0, gj_tile + q0 * 32 + 8 * (lane & 3), lane, Mrows, Ncols,
                                 pre_h, pre_l);
                else
                    sym_load_half<ph>(md, td.tm != td.tn, gi0 + lane, gj_tile, q0, 0, Mrows, Ncols, pre_e, pre_dq);
            }
            bool ok = true;
            if (lane == 0) ok = wait_bounded(tfull0 + 8 * acc, acc_phase, abort_flag, status);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) break;
            tc_fence_after();
            const float sg = (iter == 0) ? s[td.mat] : 1.0f;
            const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16) + acc * BN;
            float (*stg)[kStgW] = reinterpret_cast<float (*)[kStgW]>(stg_all + (warp - 2) * 32 * kStgW);
            if (live) {
                if constexpr (gemm) {
                    if (iter == 0)
                        epilogue_x_warp<true>(md, iter, sc, sg, gi0, gj_tile, q0, q1, Mrows, Ncols, trow, stg, lane,
                                              pre_h, pre_l);
                    else
                        epilogue_x_warp<false>(md, iter, sc, sg, gi0, gj_tile, q0, q1, Mrows, Ncols, trow, stg, lane,
                                               pre_h, pre_l);
                } else {
                    epilogue_sym_warp<ph>(md, sc, sg, td.tm != td.tn, gi0, gj_tile, q0, q1, Mrows, Ncols, trow, stg,
                                          lane, pre_e, pre_dq);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (CG == 2) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
                else mbar_arrive(tempty0 + 8 * acc);
            }
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (CG == 2) cluster_sync();     // neither CTA frees TMEM or exits while its peer may still use it
    if (warp == 1) {
        tc_fence_after();
        if (CG == 2)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                         : "memory");
    }
}

// ---------------------------------------------------------------------------
// Self-test of the bounded wait: one thread waits on an mbarrier that nothing
// ever arrives on, with the engine's wait helper and a caller-given limit.  The
// wait gives up, records MFSDP_ERR_TIMEOUT in the status word and the kernel
// returns normally; the barrier is invalidated before the CTA exits.
// ---------------------------------------------------------------------------
__global__ void bounded_wait_selftest_kernel(unsigned long long limit_ns, int32_t* status) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(smem_u32(&bar), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        (void)wait_bounded(smem_u32(&bar), 0, &abort_flag, status, limit_ns);
        asm volatile("mbarrier.inval.shared::cta.b64 [%0];" ::"r"(smem_u32(&bar)) : "memory");
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// MN-major view for 3D loads: element (k, n) of a row-major [rows][ld] matrix as
// (n % 64, k, n / 64); box {64, 64, chunks}.  The last chunk may run past column
// `cols` (into the next row or the region's slack): those values only reach output
// columns or rows past the matrix, which the epilogue discards.
bool encode_3d_mn(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld_elems, uint32_t chunks) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {64, rows, (cols + 63) / 64};
    const cuuint64_t strides[2] = {ld_elems * 2, 128};
    const cuuint32_t box[3] = {64, 64, chunks};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer, uint64_t ld_elems,
               uint32_t box_inner, uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {ld_elems * 2};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(unsigned long long limit_ns, cudaStream_t st) {
    bounded_wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns, device_status_ptr());
    return cudaGetLastError();
}

size_t tc_maps_bytes(size_t nmats) { return nmats * sizeof(TcMaps); }

int tc_tile_rows() { return TcCfg<kCtaGroup>::TILE_M; }
int tc_tile_cols() { return BN; }

bool tc_encode_maps(const std::vector<MatDev>& mats, void* host_out) {
    TcMaps* out = static_cast<TcMaps*>(host_out);
    for (size_t i = 0; i < mats.size(); ++i) {
        const MatDev& m = mats[i];
        TcMaps& mp = out[i];
        for (int b = 0; b < 2; ++b) {
            if (!encode_2d(&mp.xk[b], m.xb[b], m.c, m.r, m.ldx, BK, BM)) return false;
            if (!encode_3d_mn(&mp.xm[b], m.xb[b], m.c, m.r, m.ldx, TcCfg<kCtaGroup>::B_ROWS / 64)) return false;
        }
        if (!encode_2d(&mp.ea, m.ab, m.r, m.r, m.lda, BK, BM)) return false;
        if (!encode_2d(&mp.eb, m.bm, m.r, m.r, m.lda, BK, BM)) return false;
        if (!encode_3d_mn(&mp.eat, m.ab, m.r, m.r, m.lda, 2)) return false;
        if (!encode_3d_mn(&mp.ebt, m.bm, m.r, m.r, m.lda, 2)) return false;
    }
    return true;
}

namespace {

// Longest-processing-time assignment of a sorted tile list to nclusters
// clusters: each tile goes to the cluster with the least work so far (lowest
// id on ties), and every cluster keeps its tiles in list order.  A tile's
// work is its K depth in 64-deep blocks, but at least the epilogue's cost
// in the same units (the epilogue of one tile overlaps the next tile's MMAs,
// so a short tile still costs about one epilogue), plus one block of fixed
// overhead.  The list is rewritten cluster by cluster and seg gets the
// nclusters + 1 segment offsets.
void partition_lpt(std::vector<TileDev>& tiles, int nclusters, int epi_blocks, std::vector<int32_t>& seg) {
    nclusters = std::max(1, nclusters);
    std::vector<std::vector<TileDev>> per(static_cast<size_t>(nclusters));
    using Load = std::pair<int64_t, int>;
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int c = 0; c < nclusters; ++c) heap.push({0, c});
    for (const TileDev& t : tiles) {
        const Load l = heap.top();
        heap.pop();
        per[l.second].push_back(t);
        heap.push({l.first + std::max(t.kblk, epi_blocks) + 1, l.second});
    }
    seg.assign(static_cast<size_t>(nclusters) + 1, 0);
    tiles.clear();
    for (int c = 0; c < nclusters; ++c) {
        tiles.insert(tiles.end(), per[c].begin(), per[c].end());
        seg[c + 1] = static_cast<int32_t>(tiles.size());
    }
}

}  // namespace

int tc_launch_clusters(int ntiles, int max_clusters) { return std::max(1, std::min(ntiles, max_clusters)); }

void tc_build_tiles(const std::vector<MatDev>& mats, int max_clusters, std::vector<TileDev>& gram,
                    std::vector<TileDev>& poly, std::vector<TileDev>& gen, std::vector<int32_t>& gram_seg,
                    std::vector<int32_t>& poly_seg, std::vector<int32_t>& gen_seg) {
    constexpr int TM = TcCfg<kCtaGroup>::TILE_M;
    for (int32_t mi = 0; mi < static_cast<int32_t>(mats.size()); ++mi) {
        const MatDev& m = mats[mi];
        const int tm_n = (m.r + TM - 1) / TM;
        const int tn_sym = (m.r + BN - 1) / BN;
        const int tn_gen = (m.c + BN - 1) / BN;
        for (int i = 0; i < tm_n; ++i) {
            for (int j = 0; j < tn_sym; ++j) {
                // keep tiles that reach the upper triangle (first row <= last column of the tile)
                if (i * TM > j * BN + BN - 1) continue;
                gram.push_back({mi, i, j, (m.c + BK - 1) / BK});
                poly.push_back({mi, i, j, (m.r + BK - 1) / BK});
            }
            for (int j = 0; j < tn_gen; ++j) gen.push_back({mi, i, j, (m.r + BK - 1) / BK});
        }
    }
    // longest first; ties keep a matrix's tiles together (L2 reuse of its operands)
    auto lpt = [](const TileDev& a, const TileDev& b) {
        if (a.kblk != b.kblk) return a.kblk > b.kblk;
        if (a.mat != b.mat) return a.mat < b.mat;
        if (a.tm != b.tm) return a.tm < b.tm;
        return a.tn < b.tn;
    };
    // APPLY: column blocks outer, so that a wave of CTAs shares one slice of X
    // and the whole (small) E_B instead of streaming all of X per wave
    auto lpt_cols = [](const TileDev& a, const TileDev& b) {
        if (a.kblk != b.kblk) return a.kblk > b.kblk;
        if (a.mat != b.mat) return a.mat < b.mat;
        if (a.tn != b.tn) return a.tn < b.tn;
        return a.tm < b.tm;
    };
    std::stable_sort(gram.begin(), gram.end(), lpt);
    std::stable_sort(poly.begin(), poly.end(), lpt);
    std::stable_sort(gen.begin(), gen.end(), lpt_cols);
    // epilogue cost per tile in K blocks (measured order of magnitude): GRAM
    // stores one bf16 tile, POLY also reads one, APPLY reads and writes X's
    // two bf16 parts
    partition_lpt(gram, tc_launch_clusters(static_cast<int>(gram.size()), max_clusters), 4, gram_seg);
    partition_lpt(poly, tc_launch_clusters(static_cast<int>(poly.size()), max_clusters), 6, poly_seg);
    partition_lpt(gen, tc_launch_clusters(static_cast<int>(gen.size()), max_clusters), 10, gen_seg);
}

namespace {

constexpr int kMaxDevices = 64;

cudaLaunchConfig_t phase_config(int clusters, cudaStream_t st, cudaLaunchAttribute* attr) {
    constexpr int CG = kCtaGroup;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(clusters * CG, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = TcCfg<CG>::SMEM_BYTES;
    cfg.stream = st;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// Per device, once: the phase kernels' shared-memory attribute, then the
// number of CTA-pair clusters that fit on the device at once (the persistent
// grid).  0 on error.
int device_clusters() {
    static std::atomic<int> cached[kMaxDevices];   // zero-initialised: unknown
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        cudaGetLastError();
        return 0;
    }
    int n = cached[dev].load(std::memory_order_acquire);
    if (n > 0) return n;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    n = cached[dev].load(std::memory_order_acquire);
    if (n > 0) return n;
    constexpr int CG = kCtaGroup;
    const int smem = TcCfg<CG>::SMEM_BYTES;
    if (cudaFuncSetAttribute(tc_phase_kernel<PH_GRAM, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(tc_phase_kernel<PH_POLY, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(tc_phase_kernel<PH_APPLY, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess ||
        cudaFuncSetAttribute(tc_phase_kernel<PH_FINAL, CG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return 0;
    }
    // the four phase kernels share one launch shape (threads, shared memory, cluster)
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = phase_config(sms / CG, nullptr, attr);
    if (cudaOccupancyMaxActiveClusters(&n, tc_phase_kernel<PH_APPLY, CG>, &cfg) != cudaSuccess || n <= 0) {
        cudaGetLastError();
        n = sms / CG;
    }
    cached[dev].store(n, std::memory_order_release);
    return n;
}

template <int ph>
cudaError_t launch_phase(const MatDev* d_mats, const TcMaps* maps, int32_t nmats, const TileDev* d_tiles,
                         const int32_t* d_seg, int32_t clusters, int32_t iter, int32_t ring, const StepScalars& sc,
                         const float* s, cudaStream_t st) {
    constexpr int CG = kCtaGroup;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = phase_config(clusters, st, attr);
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, tc_phase_kernel<ph, CG>, d_mats, maps, nmats, d_tiles, d_seg, iter, ring, sc, s,
                              device_status_ptr());
}

}  // namespace

int tc_max_clusters() { return device_clusters(); }

// The ring depth a phase launch cycles through.  Under the power cap (long
// launches over operands resident in L2) four stages keep the MMAs fed, and
// fewer loads in flight per SM load the L2 less; three starve them.  Five
// stages pay where the mainloop needs more latency cover: an operand larger
// than L2 streams from DRAM, and a GRAM or APPLY launch of fewer than 16 tiles
// per cluster ends before the power cap lowers the clock.  Operand bytes: X (r x c) for
// GRAM and APPLY / FINAL, E_A (r x r) for POLY.  Same box, ring 3 / 4 / 5:
// skew 109.4 / 104.7 / 109.3 ms, 7B share 56.5 / 52.0 / 52.0 ms; block 2.18 /
// 2.00 / 1.94 ms; 32B share (its X, 283 MB, from DRAM) - / 35.1 / 34.3 ms.
int tc_ring_depth(Phase ph, const std::vector<MatDev>& mats, int64_t tiles, int32_t clusters) {
    static std::atomic<int64_t> l2_cached[kMaxDevices];   // zero: unknown
    int dev = 0;
    int64_t l2 = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
        l2 = l2_cached[dev].load(std::memory_order_acquire);
        if (l2 <= 0) {
            int v = 0;
            if (cudaDeviceGetAttribute(&v, cudaDevAttrL2CacheSize, dev) == cudaSuccess && v > 0) {
                l2 = v;
                l2_cached[dev].store(l2, std::memory_order_release);
            }
        }
    }
    cudaGetLastError();
    constexpr int deep = TcCfg<kCtaGroup>::STAGES;
    if (l2 <= 0) return deep;
    int64_t most = 0;
    for (const MatDev& m : mats) {
        const int64_t bytes = static_cast<int64_t>(m.r) * (ph == PH_POLY ? m.r : m.c) * 2;
        most = std::max(most, bytes);
    }
    // POLY's short launches keep four (block workload: POLY 0.425 -> 0.414 ms per step)
    const bool short_launch = ph != PH_POLY && tiles < 16 * static_cast<int64_t>(clusters);
    return (most > l2 || short_launch) ? deep : 4;
}

cudaError_t launch_gemm_tc(Phase ph, const MatDev* d_mats, const void* d_maps, int32_t nmats,
                           const TileDev* d_tiles, const int32_t* d_seg, int32_t clusters, int32_t iter, int32_t ring,
                           const StepScalars& sc, const float* s, cudaStream_t st) {
    if (clusters <= 0) return cudaSuccess;
    if (device_clusters() <= 0) return cudaErrorInvalidConfiguration;   // attributes not set on this device
    const TcMaps* maps = static_cast<const TcMaps*>(d_maps);
    cudaError_t e;
    switch (ph) {
        case PH_GRAM: e = launch_phase<PH_GRAM>(d_mats, maps, nmats, d_tiles, d_seg, clusters, iter, ring, sc, s, st); break;
        case PH_POLY: e = launch_phase<PH_POLY>(d_mats, maps, nmats, d_tiles, d_seg, clusters, iter, ring, sc, s, st); break;
        case PH_APPLY: e = launch_phase<PH_APPLY>(d_mats, maps, nmats, d_tiles, d_seg, clusters, iter, ring, sc, s, st); break;
        default: e = launch_phase<PH_FINAL>(d_mats, maps, nmats, d_tiles, d_seg, clusters, iter, ring, sc, s, st); break;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace mfsdp
